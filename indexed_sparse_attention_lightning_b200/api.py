"""Python binding over ``libsa.so``.

Argument marshalling only: torch tensors (device memory, streams) are turned
into the C structs of ``include/sa.h`` and passed to the library, which runs
every step of the path in its own CUDA kernels.  Nothing here computes.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import _abi
from ._abi import SaCache, SaError, SaNewTokens, SaQuery, check

_TORCH_RAW = {np.dtype(np.uint8): torch.uint8, np.dtype(np.uint16): torch.int16,
              np.dtype(np.float32): torch.float32, np.dtype(np.int32): torch.int32}


def _t(a: Optional[np.ndarray], device) -> Optional[torch.Tensor]:
    """numpy -> torch on `device`, raw bits preserved (bf16 travels as int16)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t, name: str, dtype=None, shape=None, optional: bool = False) -> None:
    """Marshalling precondition: a contiguous CUDA tensor (of `dtype` and `shape`
    when given).  The library reads raw pointers, so a host tensor, a strided
    view or an int64 index tensor would be misread; refuse them here."""
    if t is None:
        if optional:
            return
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} has dtype {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}, "
                                               f"expected {tuple(shape)}")


def _need_rows(t, name: str, n_rows: int, min_cols: int) -> None:
    """A CUDA fp32 matrix whose rows may be padded (unit column stride)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if t.dtype != torch.float32 or t.dim() != 2 or t.stride(1) != 1:
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} must be a float32 matrix with unit "
                                               "column stride")
    if t.shape[0] != n_rows or t.shape[1] < min_cols:
        raise SaError(_abi.SA_ERR_INVALID_ARG, f"{name} has shape {tuple(t.shape)}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


@dataclass
class DeviceCache:
    """The paged index-key and latent caches of one layer, resident on the device."""

    page_table: torch.Tensor
    seq_len: torch.Tensor
    num_pages: int
    index_dtype: str
    k_index: torch.Tensor
    k_index_scale: Optional[torch.Tensor]
    kv_dtype: str
    kv: torch.Tensor
    kv_rope: Optional[torch.Tensor]
    kv_scale: Optional[torch.Tensor]
    d_index: int
    d_latent: int
    d_rope: int
    page_size: int = 64
    kv_scale_tile: tuple = (0, 0)   # (tokens, dims) per e4m3 scale; (0, 0): one per page

    def struct(self) -> SaCache:
        _need(self.page_table, "page_table", torch.int32)
        _need(self.seq_len, "seq_len", torch.int32)
        for name in ("k_index", "k_index_scale", "kv", "kv_rope", "kv_scale"):
            _need(getattr(self, name), name, optional=True)
        return SaCache(
            page_table=_ptr(self.page_table), seq_len=_ptr(self.seq_len),
            batch=self.page_table.shape[0], max_pages=self.page_table.shape[1],
            num_pages=self.num_pages, page_size=self.page_size,
            index_dtype=_abi.DTYPES[self.index_dtype], k_index=_ptr(self.k_index),
            k_index_scale=_ptr(self.k_index_scale), d_index=self.d_index,
            kv_dtype=_abi.DTYPES[self.kv_dtype], kv=_ptr(self.kv), kv_rope=_ptr(self.kv_rope),
            kv_scale=_ptr(self.kv_scale), d_latent=self.d_latent, d_rope=self.d_rope,
            kv_scale_tokens=int(self.kv_scale_tile[0]), kv_scale_dims=int(self.kv_scale_tile[1]))


@dataclass
class DeviceQueries:
    """One step's query tokens (indexer query, head weights, attention query)."""

    q_seq: torch.Tensor
    q_pos: torch.Tensor
    max_visible: int
    q_index: torch.Tensor
    q_index_scale: Optional[torch.Tensor]
    w: torch.Tensor
    h_index: int
    q_dtype: str
    q: torch.Tensor
    heads: int
    sm_scale: float
    # chunked prefill: queries 4i .. 4i+3 belong to one sequence (see sa_query.q_group)
    q_group: int = 1

    @property
    def n_q(self) -> int:
        return int(self.q_seq.shape[0])

    def struct(self) -> SaQuery:
        _need(self.q_seq, "q_seq", torch.int32)
        _need(self.q_pos, "q_pos", torch.int32)
        for name in ("q_index", "q_index_scale", "w", "q"):
            _need(getattr(self, name), name, optional=True)
        return SaQuery(
            n_q=self.n_q, q_seq=_ptr(self.q_seq), q_pos=_ptr(self.q_pos),
            max_visible=self.max_visible, q_index=_ptr(self.q_index),
            q_index_scale=_ptr(self.q_index_scale), w=_ptr(self.w), h_index=self.h_index,
            q_dtype=_abi.DTYPES[self.q_dtype], q=_ptr(self.q), heads=self.heads,
            sm_scale=self.sm_scale, q_group=self.q_group)

    def tensors(self) -> dict:
        return {"q_seq": self.q_seq, "q_pos": self.q_pos, "q_index": self.q_index,
                "q_index_scale": self.q_index_scale, "w": self.w, "q": self.q}

    def copy_from(self, host: dict, non_blocking: bool = True) -> int:
        """Copy a step's inputs (e.g. pinned host tensors) into these buffers.
        Returns the bytes copied."""
        n = 0
        for k, dst in self.tensors().items():
            src = host.get(k)
            if dst is None or src is None:
                continue
            dst.copy_(src, non_blocking=non_blocking)
            n += src.numel() * src.element_size()
        return n


def upload(wl, device="cuda") -> tuple[DeviceCache, DeviceQueries]:
    """Place a workload (numpy arrays) on the device."""
    sp = wl.spec
    if getattr(sp, "index_scale_group", 0):
        raise SaError(_abi.SA_ERR_UNSUPPORTED,
                      "upload: fp32 index scales per group of values have no kernel in this "
                      "library (its group-scaled index format is MXFP8: E8M0 scales per 32)")
    cache = DeviceCache(
        page_table=_t(wl.page_table, device), seq_len=_t(wl.seq_len, device),
        num_pages=int(wl.num_pages), index_dtype=sp.index_dtype,
        k_index=_t(wl.k_index, device), k_index_scale=_t(wl.k_index_scale, device),
        kv_dtype=sp.kv_dtype, kv=_t(wl.kv, device), kv_rope=_t(wl.kv_rope, device),
        kv_scale=_t(wl.kv_scale, device), d_index=sp.d_index, d_latent=sp.d_latent,
        d_rope=sp.d_rope, page_size=sp.page_size, kv_scale_tile=tuple(sp.kv_scale_tile))
    queries = DeviceQueries(
        q_seq=_t(wl.q_seq, device), q_pos=_t(wl.q_pos, device), max_visible=wl.max_visible,
        q_index=_t(wl.q_index, device), q_index_scale=_t(wl.q_index_scale, device),
        w=_t(wl.w, device), h_index=sp.h_index, q_dtype=sp.q_dtype, q=_t(wl.q, device),
        heads=sp.heads, sm_scale=sp.softmax_scale,
        q_group=4 if sp.queries[0] == "prefill" else 1)
    return cache, queries


def host_queries(wl, pin: bool = True) -> dict:
    """A step's query inputs as (pinned) host tensors, for end-to-end timing."""
    out = {}
    for k in ("q_seq", "q_pos", "q_index", "q_index_scale", "w", "q"):
        a = getattr(wl, k)
        if a is None:
            continue
        t = _t(a, "cpu")
        out[k] = t.pin_memory() if pin else t
    return out


# ---------------------------------------------------------------- workspace ---

def workspace_size(cache: DeviceCache, queries: DeviceQueries, top_k: int, uses: int) -> int:
    c, q = cache.struct(), queries.struct()
    n = _abi.lib().sa_workspace_size(ctypes.byref(c), ctypes.byref(q), top_k, uses)
    if n == 0:
        raise SaError(_abi.SA_ERR_INVALID_ARG, "sa_workspace_size")
    return int(n)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Device workspace (torch allocations are at least 256-byte aligned)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def device_status(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    """(status, detail) of the last call that used `ws`; synchronises the stream."""
    detail = ctypes.c_int32(0)
    st = _abi.lib().sa_device_status(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


# -------------------------------------------------------------- entry points ---

def indexer_score(cache: DeviceCache, queries: DeviceQueries, scores=None, ws=None,
                  stream=None) -> torch.Tensor:
    dev = queries.q_seq.device
    if scores is None:
        scores = torch.full((queries.n_q, max(1, queries.max_visible)), float("nan"),
                            dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(workspace_size(cache, queries, 1, _abi.SA_WS_INDEXER), dev)
    _need_rows(scores, "scores", queries.n_q, queries.max_visible)
    _need(ws, "ws")
    c, q = cache.struct(), queries.struct()
    check(_abi.lib().sa_indexer_score(ctypes.byref(c), ctypes.byref(q), _ptr(scores),
                                      scores.stride(0), _ptr(ws), ws.numel(), _stream(stream)),
          "sa_indexer_score")
    return scores


def topk(scores: torch.Tensor, valid_len: torch.Tensor, top_k: int, max_valid: int,
         idx=None, ws=None, stream=None) -> torch.Tensor:
    n_q = scores.shape[0]
    if idx is None:
        idx = torch.empty((n_q, top_k), dtype=torch.int32, device=scores.device)
    if ws is None:
        ws = workspace(256, scores.device)
    _need_rows(scores, "scores", n_q, max_valid)
    _need(valid_len, "valid_len", torch.int32, (n_q,))
    _need(idx, "idx", torch.int32, (n_q, top_k))
    _need(ws, "ws")
    check(_abi.lib().sa_topk(_ptr(scores), scores.stride(0), _ptr(valid_len), n_q, max_valid,
                             top_k, _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)),
          "sa_topk")
    return idx


def _outputs(queries: DeviceQueries, d_latent: int, out, lse, out_dtype: str):
    dev = queries.q_seq.device
    dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    if out is None:
        out = torch.empty((queries.n_q, queries.heads, d_latent), dtype=dt, device=dev)
    if lse is None:
        lse = torch.empty((queries.n_q, queries.heads), dtype=torch.float32, device=dev)
    _need(out, "out", dt, (queries.n_q, queries.heads, d_latent))
    _need(lse, "lse", torch.float32, (queries.n_q, queries.heads))
    return out, lse


def sparse_mla_attn(cache: DeviceCache, queries: DeviceQueries, idx: torch.Tensor, top_k: int,
                    out=None, lse=None, out_dtype: str = "bf16", ws=None, stream=None):
    out, lse = _outputs(queries, cache.d_latent, out, lse, out_dtype)
    if ws is None:
        ws = workspace(workspace_size(cache, queries, top_k, _abi.SA_WS_ATTN), idx.device)
    _need(idx, "idx", torch.int32, (queries.n_q, top_k))
    _need(ws, "ws")
    c, q = cache.struct(), queries.struct()
    check(_abi.lib().sa_sparse_mla_attn(ctypes.byref(c), ctypes.byref(q), _ptr(idx), top_k,
                                        _ptr(out), _abi.DTYPES[out_dtype], _ptr(lse), _ptr(ws),
                                        ws.numel(), _stream(stream)),
          "sa_sparse_mla_attn")
    return out, lse


def decode(cache: DeviceCache, queries: DeviceQueries, top_k: int, out=None, lse=None,
           idx=None, out_dtype: str = "bf16", ws=None, stream=None, phase_events=None):
    """Fused indexer -> top-K -> sparse attention.  Returns (out, lse, idx-or-None).

    ``phase_events``: optional list of len(_abi.DECODE_PHASES) + 1 torch.cuda.Event
    objects recorded at the phase boundaries (sa_decode_traced)."""
    out, lse = _outputs(queries, cache.d_latent, out, lse, out_dtype)
    if ws is None:
        ws = workspace(workspace_size(cache, queries, top_k, _abi.SA_WS_DECODE),
                       queries.q_seq.device)
    _need(idx, "idx", torch.int32, (queries.n_q, top_k), optional=True)
    _need(ws, "ws")
    c, q = cache.struct(), queries.struct()
    args = (ctypes.byref(c), ctypes.byref(q), top_k, _ptr(idx), _ptr(out),
            _abi.DTYPES[out_dtype], _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    if phase_events is None:
        check(_abi.lib().sa_decode(*args), "sa_decode")
    else:
        if len(phase_events) != len(_abi.DECODE_PHASES) + 1:
            raise ValueError("need one event per phase boundary")
        for e in phase_events:
            if e.cuda_event == 0:       # torch creates the CUDA event on first record
                e.record(stream if stream is not None else torch.cuda.current_stream())
        handles = (ctypes.c_void_p * len(phase_events))(*[e.cuda_event for e in phase_events])
        check(_abi.lib().sa_decode_traced(*args, handles), "sa_decode_traced")
    return out, lse, idx


# -------------------------------------------- context-parallel decode steps ---

def local_candidates(cache: DeviceCache, queries: DeviceQueries, top_k: int,
                     offset: torch.Tensor, score=None, pos=None, ws=None, stream=None):
    """This GPU's top_k of its context shard as (score fp32, position + offset
    int32), both [n_q, top_k], ascending positions, (-inf, -1) padding."""
    dev = queries.q_seq.device
    n_q = queries.n_q
    if score is None:
        score = torch.empty((n_q, top_k), dtype=torch.float32, device=dev)
    if pos is None:
        pos = torch.empty((n_q, top_k), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(workspace_size(cache, queries, top_k, _abi.SA_WS_DECODE), dev)
    _need(offset, "offset", torch.int32, (n_q,))
    _need(score, "score", torch.float32, (n_q, top_k))
    _need(pos, "pos", torch.int32, (n_q, top_k))
    _need(ws, "ws")
    c, q = cache.struct(), queries.struct()
    check(_abi.lib().sa_local_candidates(ctypes.byref(c), ctypes.byref(q), top_k, _ptr(offset),
                                         _ptr(score), _ptr(pos), _ptr(ws), ws.numel(),
                                         _stream(stream)),
          "sa_local_candidates")
    return score, pos, ws


def merge_candidates(score: torch.Tensor, pos: torch.Tensor, top_k: int, lo: torch.Tensor,
                     hi: torch.Tensor, idx_global=None, idx_local=None, stream=None):
    """All ranks' candidates [n_ranks, n_q, top_k] -> (global top-K positions,
    the ones in [lo, hi) as local positions), both int32 [n_q, top_k]."""
    n_ranks, n_q, k = score.shape
    if k != top_k:
        raise SaError(_abi.SA_ERR_INVALID_ARG, "merge_candidates: candidate rows of top_k")
    _need(score, "score", torch.float32, (n_ranks, n_q, top_k))
    _need(pos, "pos", torch.int32, (n_ranks, n_q, top_k))
    _need(lo, "lo", torch.int32, (n_q,))
    _need(hi, "hi", torch.int32, (n_q,))
    if idx_global is None:
        idx_global = torch.empty((n_q, top_k), dtype=torch.int32, device=score.device)
    if idx_local is None:
        idx_local = torch.empty((n_q, top_k), dtype=torch.int32, device=score.device)
    _need(idx_global, "idx_global", torch.int32, (n_q, top_k))
    _need(idx_local, "idx_local", torch.int32, (n_q, top_k))
    check(_abi.lib().sa_merge_candidates(_ptr(score), _ptr(pos), n_ranks, n_q, top_k, _ptr(lo),
                                         _ptr(hi), _ptr(idx_global), _ptr(idx_local),
                                         _stream(stream)),
          "sa_merge_candidates")
    return idx_global, idx_local


def combine_partials(o_part: torch.Tensor, lse_part: torch.Tensor, out=None, lse=None,
                     out_dtype: str = "bf16", stream=None):
    """Partial outputs [n_parts, n_q, heads, d] (fp32) with their lse [n_parts,
    n_q, heads] -> (out [n_q, heads, d], lse [n_q, heads])."""
    n_parts, n_q, heads, d = o_part.shape
    _need(o_part, "o_part", torch.float32, (n_parts, n_q, heads, d))
    _need(lse_part, "lse_part", torch.float32, (n_parts, n_q, heads))
    dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    if out is None:
        out = torch.empty((n_q, heads, d), dtype=dt, device=o_part.device)
    if lse is None:
        lse = torch.empty((n_q, heads), dtype=torch.float32, device=o_part.device)
    _need(out, "out", dt, (n_q, heads, d))
    _need(lse, "lse", torch.float32, (n_q, heads))
    check(_abi.lib().sa_combine_partials(_ptr(o_part), _ptr(lse_part), n_parts, n_q, heads, d,
                                         _ptr(out), _abi.DTYPES[out_dtype], _ptr(lse),
                                         _stream(stream)),
          "sa_combine_partials")
    return out, lse


# ------------------------------------------------------- input preparation ---

_IN_DTYPES = {torch.bfloat16: "bf16", torch.float32: "f32"}


def _in_dtype(t: torch.Tensor) -> int:
    if t.dtype not in _IN_DTYPES:
        raise SaError(_abi.SA_ERR_UNSUPPORTED, "input dtype (bfloat16 or float32)")
    return _abi.DTYPES[_IN_DTYPES[t.dtype]]


def quantize_index_query(q: torch.Tensor, out=None, scale=None, stream=None):
    """Indexer query [n_q, h_index, d_index] (bfloat16 or float32) -> (e4m3 codes
    uint8 [n_q, h_index, d_index], fp32 scales [n_q, h_index])."""
    _need(q, "q", (torch.bfloat16, torch.float32))
    n_q, h, d = q.shape
    if out is None:
        out = torch.empty((n_q, h, d), dtype=torch.uint8, device=q.device)
    if scale is None:
        scale = torch.empty((n_q, h), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.uint8, (n_q, h, d))
    _need(scale, "scale", torch.float32, (n_q, h))
    check(_abi.lib().sa_quantize_index_query(_ptr(q), _in_dtype(q), n_q, h, d, _ptr(out),
                                             _ptr(scale), _stream(stream)),
          "sa_quantize_index_query")
    return out, scale


def append_tokens(cache: DeviceCache, seq: torch.Tensor, pos: torch.Tensor,
                  k_index: Optional[torch.Tensor] = None, kv: Optional[torch.Tensor] = None,
                  ws=None, stream=None) -> torch.Tensor:
    """Write new tokens (sequence, position) into the cache's pools in place:
    index keys [n_new, d_index] and latent + rope rows [n_new, d_latent + d_rope],
    both bfloat16 or both float32 (either may be None).  Returns the workspace,
    whose status word records skipped tokens (see device_status)."""
    ins = [t for t in (k_index, kv) if t is not None]
    if len({t.dtype for t in ins}) > 1:
        raise SaError(_abi.SA_ERR_INVALID_ARG, "append_tokens: k_index and kv dtypes differ")
    n_new = int(seq.numel())
    _need(seq, "seq", torch.int32, (n_new,))
    _need(pos, "pos", torch.int32, (n_new,))
    _need(k_index, "k_index", (torch.bfloat16, torch.float32), (n_new, cache.d_index),
          optional=True)
    _need(kv, "kv", (torch.bfloat16, torch.float32), (n_new, cache.d_latent + cache.d_rope),
          optional=True)
    dt = _in_dtype(ins[0]) if ins else _abi.SA_BF16
    c = cache.struct()
    if ws is None:
        n = _abi.lib().sa_workspace_size(ctypes.byref(c), None, 0, _abi.SA_WS_APPEND)
        if n == 0:
            raise SaError(_abi.SA_ERR_INVALID_ARG, "sa_workspace_size")
        ws = workspace(n, seq.device)
    _need(ws, "ws")
    t = SaNewTokens(n_new=n_new, seq=_ptr(seq), pos=_ptr(pos), in_dtype=dt,
                    k_index=_ptr(k_index), kv=_ptr(kv))
    check(_abi.lib().sa_append_tokens(ctypes.byref(c), ctypes.byref(t), _ptr(ws), ws.numel(),
                                      _stream(stream)),
          "sa_append_tokens")
    return ws
