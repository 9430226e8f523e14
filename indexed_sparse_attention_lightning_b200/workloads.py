"""Seeded synthetic workloads for the indexed sparse attention path.

This module draws random numbers, rounds them into the storage formats the path
reads (e4m3 codes with fp32 scales, bf16, fp32) and lays them out in a paged
cache.  It holds none of the method's arithmetic: nothing here scores, selects
or attends.  The CPU oracle (under ``oracle/``) and the CUDA path both consume
the arrays it returns, so the two sides see identical bytes.

Cache layout (the pages describe the cache as paged and read in place by the
indexer and the sparse attention kernel -- "Optimizing Next-Gen LLM Inference"
§3.1/§3.3, "Inference Acceleration for New Large Model Architectures" §3.1):

* ``page_table[b, i]`` is the physical page holding tokens ``64*i .. 64*i+63``
  of sequence ``b``; entries past the sequence end are -1.
* index keys ``k_index[P, 64, d_index]`` (fp32, bf16, or e4m3 codes with one
  fp32 scale per token in ``k_index_scale[P, 64]``, or one per group of values
  in ``k_index_scale[P, 64, d_index / group]``; or MXFP8: e4m3 codes with one
  E8M0 scale byte per 32 values in ``k_index_scale[P, 64, d_index / 32]``,
  uint8);
* MLA latent rows ``kv[P, 64, d_latent + d_rope]`` (fp32 or bf16), or for the
  FP8 cache ``kv[P, 64, d_latent]`` e4m3 codes, ``kv_scale[P, 64 / ts, d_latent / td]``
  (one fp32 scale per tile of ts tokens x td latent dims of a page; the default
  (64, d_latent) is one per page) and ``kv_rope[P, 64, d_rope]`` bf16.

Slots past a sequence's end and pages no sequence owns are filled with NaN, so
that any read outside the visible range shows up as NaN in a result.

Quantisation rule (inputs arrive already quantised): ``scale = amax / 448``
(1 when amax is 0), ``code = RNE(x / scale)`` saturated to +-448 in e4m3fn.
MXFP8 (OCP MX rule, power-of-two scales): per group of 32 values
``scale = 2^(floor(log2 amax) - 8)`` (8 = the exponent of e4m3's largest
value), stored as the E8M0 byte ``127 + floor(log2 amax) - 8``; codes as above
(values that land in [448, 512) of the scale saturate to 448); an all-zero
group stores byte 127 (scale 1).
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0
E4M3_NAN = 0x7F
BF16_NAN = 0x7FC0

# ----------------------------------------------------------------------------
# Specs
# ----------------------------------------------------------------------------


@dataclass(frozen=True)
class WorkloadSpec:
    """Shape, dtype and structure of one synthetic workload."""

    name: str
    seed: int
    batch: int
    seq_len: tuple                 # ("fixed", L), ("uniform", lo, hi) inclusive, ("list", (L0, L1, ...))
    queries: tuple = ("decode",)   # ("decode",) or ("prefill", first_pos, count)
    h_index: int = 64
    d_index: int = 128
    index_dtype: str = "e4m3"      # "e4m3", "mxfp8", "bf16" or "f32"
    # e4m3 index scales: 0 = one per key row and one per (query, head) row; g = one
    # per g consecutive values of a row (the pages' group-32 quantisation)
    index_scale_group: int = 0
    top_k: int = 2048
    heads: int = 128
    d_latent: int = 512
    d_rope: int = 64
    kv_dtype: str = "bf16"         # "f32", "bf16" or "e4m3"
    q_dtype: str = "bf16"          # "f32" or "bf16"
    page_size: int = 64
    paging: str = "permuted"       # "identity" or "permuted"
    keys: tuple = ("iid",)         # ("iid",), ("planted", frac, sigma), ("clusters", n, span)
    sm_scale: Optional[float] = None  # default 1/sqrt(d_latent + d_rope)
    # e4m3 latent cache: one fp32 scale per tile of (tokens of a page, latent
    # dims); (0, 0) is one scale per page
    kv_scale_tile: tuple = (0, 0)
    poison_pages: int = 2

    @property
    def d_qk(self) -> int:
        return self.d_latent + self.d_rope

    @property
    def kv_tile(self) -> tuple:
        """(tokens, latent dims) covered by one e4m3 scale."""
        st, sd = self.kv_scale_tile
        return (st or self.page_size, sd or self.d_latent)

    @property
    def softmax_scale(self) -> float:
        if self.sm_scale is not None:
            return float(self.sm_scale)
        return 1.0 / math.sqrt(self.d_qk)


TINY = WorkloadSpec(
    name="tiny_decode_b1_1k_fp32", seed=0, batch=1, seq_len=("fixed", 1024),
    h_index=4, d_index=32, index_dtype="f32", top_k=64, heads=4, d_latent=64,
    d_rope=16, kv_dtype="f32", q_dtype="f32", paging="identity",
    sm_scale=1.0 / math.sqrt(80.0))

DECODE_B8_8K = WorkloadSpec(
    name="decode_b8_8k", seed=1, batch=8, seq_len=("fixed", 8192))

DECODE_B64_16K_32K = WorkloadSpec(
    name="decode_b64_16k_32k_planted", seed=2, batch=64,
    seq_len=("uniform", 16384, 32768), keys=("planted", 0.05, 3.0))

PREFILL_4096Q_64K = WorkloadSpec(
    name="prefill_4096q_64k", seed=3, batch=1, seq_len=("fixed", 65536),
    queries=("prefill", 61440, 4096))

DECODE_B2_1M_FP8KV = WorkloadSpec(
    name="decode_b2_1m_fp8kv_clustered", seed=4, batch=2,
    seq_len=("fixed", 1048576), kv_dtype="e4m3", keys=("clusters", 16, 4096))

CONFIGS = (TINY, DECODE_B8_8K, DECODE_B64_16K_32K, PREFILL_4096Q_64K,
           DECODE_B2_1M_FP8KV)

# A smaller decode case for full profiler captures: the same kernels and
# per-query work as the 64-sequence decode, at a fixed 16K context (138 MB of
# index keys, more than L2; about 1.7 GB on the device).
PROFILE_B64_16K = WorkloadSpec(
    name="profile_decode_b64_16k", seed=3, batch=64, seq_len=("fixed", 16384))

# the headline decode with the indexer's BF16 path (unquantised query and keys)
DECODE_B64_BF16_INDEX = WorkloadSpec(
    name="decode_b64_16k_32k_bf16_index", seed=2, batch=64, seq_len=("uniform", 16384, 32768),
    keys=("planted", 0.05, 3.0), index_dtype="bf16")

# the 1M FP8 decode with the pages' latent-cache granularity: one scale per
# token and per 128 latent dims instead of one per page
DECODE_B2_1M_FP8KV_TILE_1X128 = WorkloadSpec(
    name="decode_b2_1m_fp8kv_tile_1x128", seed=4, batch=2, seq_len=("fixed", 1048576),
    kv_dtype="e4m3", keys=("clusters", 16, 4096), kv_scale_tile=(1, 128))

# the headline decode with the pages' MXFP8 index path: e4m3 index query and
# keys with one power-of-two (E8M0) scale per 32 values
DECODE_B64_MXFP8_INDEX = WorkloadSpec(
    name="decode_b64_16k_32k_mxfp8_index", seed=2, batch=64, seq_len=("uniform", 16384, 32768),
    keys=("planted", 0.05, 3.0), index_dtype="mxfp8")

EXTRA = (PROFILE_B64_16K, DECODE_B64_BF16_INDEX, DECODE_B2_1M_FP8KV_TILE_1X128,
         DECODE_B64_MXFP8_INDEX)


def spec(which) -> WorkloadSpec:
    """Look a spec up by index (0..4) or by name."""
    if isinstance(which, int):
        return CONFIGS[which]
    for s in CONFIGS + EXTRA:
        if s.name == which:
            return s
    raise KeyError(which)


# ----------------------------------------------------------------------------
# Workload container
# ----------------------------------------------------------------------------


@dataclass
class Workload:
    spec: WorkloadSpec
    seq_len: np.ndarray          # int32 [B]
    page_table: np.ndarray       # int32 [B, max_pages]
    num_pages: int
    q_seq: np.ndarray            # int32 [n_q]
    q_pos: np.ndarray            # int32 [n_q]; visible length is q_pos + 1
    k_index: np.ndarray          # f32, uint16 (bf16) or uint8 (e4m3) [P, ps, d_index]
    k_index_scale: Optional[np.ndarray]  # f32 [P, ps] (or [P, ps, d_index / group])
    q_index: np.ndarray          # f32, uint16 (bf16) or uint8 (e4m3) [n_q, h_index, d_index]
    q_index_scale: Optional[np.ndarray]  # f32 [n_q, h_index] (or [n_q, h_index, d_index / group])
    w: np.ndarray                # f32 [n_q, h_index]
    kv: np.ndarray               # f32/uint16(bf16) [P, ps, d_qk] or uint8 [P, ps, d_latent]
    kv_rope: Optional[np.ndarray]  # uint16 (bf16) [P, ps, d_rope] for the e4m3 cache
    kv_scale: Optional[np.ndarray]  # f32 [P, 64 / tile tokens, d_latent / tile dims] (e4m3)
    q: np.ndarray                # f32 or uint16 (bf16) [n_q, heads, d_qk]
    planted: dict = field(default_factory=dict)  # seq -> sorted planted positions
    clusters: dict = field(default_factory=dict)  # seq -> list of (start, len)

    @property
    def n_q(self) -> int:
        return int(self.q_seq.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def visible(self) -> np.ndarray:
        return (self.q_pos.astype(np.int64) + 1).astype(np.int32)

    @property
    def max_visible(self) -> int:
        return int(self.visible.max())


# ----------------------------------------------------------------------------
# Rounding helpers (storage formats only)
# ----------------------------------------------------------------------------


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (torch's conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """fp32 -> e4m3fn codes, saturating at +-448, round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.clamp(-E4M3_MAX, E4M3_MAX)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def amax_scale(amax: np.ndarray) -> np.ndarray:
    s = (amax.astype(np.float32) / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows_e4m3(x: np.ndarray):
    """One scale per row of the last axis: returns (codes uint8, scale f32)."""
    amax = np.abs(x).max(axis=-1)
    scale = amax_scale(amax)
    return to_e4m3_codes(x / scale[..., None]), scale


def quantize_groups_e4m3(x: np.ndarray, group: int):
    """One scale per `group` consecutive values of the last axis: returns
    (codes uint8 like x, scale f32 [..., last / group])."""
    g = x.reshape(x.shape[:-1] + (x.shape[-1] // group, group))
    codes, scale = quantize_rows_e4m3(g)
    return codes.reshape(x.shape), scale


MX_GROUP = 32


def quantize_mxfp8(x: np.ndarray):
    """OCP MX quantisation of groups of 32 values of the last axis: returns
    (e4m3 codes uint8 like x, E8M0 scale bytes uint8 [..., last / 32])."""
    g = x.reshape(x.shape[:-1] + (x.shape[-1] // MX_GROUP, MX_GROUP)).astype(np.float32)
    amax = np.abs(g).max(axis=-1)
    _, ex = np.frexp(amax)                      # amax = m * 2^ex, m in [0.5, 1)
    e = np.where(amax > 0, ex.astype(np.int64) - 1 - 8, 0)  # floor(log2 amax) - 8
    byte = np.clip(e + 127, 0, 254).astype(np.uint8)
    scale = np.ldexp(np.float32(1.0), byte.astype(np.int64) - 127).astype(np.float32)
    codes = to_e4m3_codes(g / scale[..., None])
    return codes.reshape(x.shape), byte


def e8m0_value(byte: np.ndarray) -> np.ndarray:
    """E8M0 bytes -> their fp32 values 2^(b - 127) (255 -> NaN); storage decode only."""
    b = np.asarray(byte).astype(np.int64)
    v = np.ldexp(np.float64(1.0), b - 127)
    return np.where(b == 255, np.nan, v).astype(np.float32)


def _quantize_index(x: np.ndarray, group: int, mx: bool = False):
    if mx:
        return quantize_mxfp8(x)
    return quantize_groups_e4m3(x, group) if group > 0 else quantize_rows_e4m3(x)


# ----------------------------------------------------------------------------
# Generation
# ----------------------------------------------------------------------------

_CHUNK = 1 << 16  # tokens drawn per step for the large per-sequence arrays


def _seq_lengths(sp: WorkloadSpec, rng) -> np.ndarray:
    kind = sp.seq_len[0]
    if kind == "fixed":
        return np.full(sp.batch, int(sp.seq_len[1]), dtype=np.int32)
    if kind == "uniform":
        lo, hi = int(sp.seq_len[1]), int(sp.seq_len[2])
        return rng.integers(lo, hi + 1, size=sp.batch, dtype=np.int64).astype(np.int32)
    if kind == "list":
        lens = np.asarray(sp.seq_len[1], dtype=np.int32)
        if lens.shape != (sp.batch,) or lens.min() < 1:
            raise ValueError("one positive length per sequence")
        return lens
    raise ValueError(sp.seq_len)


def _queries(sp: WorkloadSpec, lens: np.ndarray):
    if sp.queries[0] == "decode":
        q_seq = np.arange(sp.batch, dtype=np.int32)
        q_pos = (lens - 1).astype(np.int32)
        return q_seq, q_pos
    if sp.queries[0] == "prefill":
        first, count = int(sp.queries[1]), int(sp.queries[2])
        if sp.batch != 1:
            raise ValueError("prefill workloads hold one sequence")
        if first + count > int(lens[0]):
            raise ValueError("prefill positions exceed the context")
        q_seq = np.zeros(count, dtype=np.int32)
        q_pos = (first + np.arange(count)).astype(np.int32)
        return q_seq, q_pos
    raise ValueError(sp.queries)


def _phys_rows(page_table_row: np.ndarray, start: int, stop: int, ps: int) -> np.ndarray:
    s = np.arange(start, stop, dtype=np.int64)
    return page_table_row[s // ps].astype(np.int64) * ps + (s % ps)


def _normal(rng, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_workload(sp: WorkloadSpec) -> Workload:
    """Draw the workload ``sp`` deterministically from ``sp.seed`` (numpy PCG64)."""
    rng = np.random.default_rng(sp.seed)
    ps = sp.page_size
    lens = _seq_lengths(sp, rng)
    pages_per_seq = (lens.astype(np.int64) + ps - 1) // ps
    n_used = int(pages_per_seq.sum())
    num_pages = n_used + sp.poison_pages
    max_pages = int(pages_per_seq.max())

    # physical placement of logical pages
    if sp.paging == "identity":
        perm = np.arange(num_pages, dtype=np.int64)
    elif sp.paging == "permuted":
        perm = rng.permutation(num_pages).astype(np.int64)
    else:
        raise ValueError(sp.paging)
    page_table = np.full((sp.batch, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(sp.batch):
        n = int(pages_per_seq[b])
        page_table[b, :n] = perm[off:off + n]
        off += n

    q_seq, q_pos = _queries(sp, lens)
    n_q = q_seq.shape[0]
    H_I, d_I = sp.h_index, sp.d_index

    # indexer queries and head weights
    qi = _normal(rng, (n_q, H_I, d_I))
    w = (_normal(rng, (n_q, H_I)) / np.float32(math.sqrt(H_I))).astype(np.float32)
    if sp.index_scale_group and (sp.index_dtype != "e4m3" or d_I % sp.index_scale_group):
        raise ValueError("group scales need e4m3 index data and a group dividing d_index")
    if sp.index_dtype == "e4m3":
        q_index, q_index_scale = _quantize_index(qi, sp.index_scale_group)
    elif sp.index_dtype == "mxfp8":
        if d_I % MX_GROUP or sp.index_scale_group:
            raise ValueError("MXFP8 needs d_index a multiple of 32 and no other scale group")
        q_index, q_index_scale = quantize_mxfp8(qi)
    elif sp.index_dtype == "bf16":
        q_index, q_index_scale = to_bf16_bits(qi), None
    elif sp.index_dtype == "f32":
        q_index, q_index_scale = qi, None
    else:
        raise ValueError(sp.index_dtype)

    # index keys
    rows = num_pages * ps
    if sp.index_dtype == "e4m3":
        k_index = np.full((rows, d_I), E4M3_NAN, dtype=np.uint8)
        k_index_scale = np.full((rows,) + ((d_I // sp.index_scale_group,)
                                           if sp.index_scale_group else ()),
                                np.nan, dtype=np.float32)
    elif sp.index_dtype == "mxfp8":
        k_index = np.full((rows, d_I), E4M3_NAN, dtype=np.uint8)
        k_index_scale = np.full((rows, d_I // MX_GROUP), 255, dtype=np.uint8)  # NaN scale
    elif sp.index_dtype == "bf16":
        k_index = np.full((rows, d_I), BF16_NAN, dtype=np.uint16)
        k_index_scale = None
    else:
        k_index = np.full((rows, d_I), np.nan, dtype=np.float32)
        k_index_scale = None

    planted, clusters = {}, {}
    for b in range(sp.batch):
        L = int(lens[b])
        kind = sp.keys[0]
        if kind == "planted":
            frac, sigma = float(sp.keys[1]), float(sp.keys[2])
            n_plant = int(round(frac * L))
            pos = np.sort(rng.choice(L, size=n_plant, replace=False)).astype(np.int64)
            planted[b] = pos
            # direction: the query's heads weighted by their positive head weights,
            # taken from the values the indexer actually sees (dequantised)
            qb = np.nonzero(q_seq == b)[0]
            if qb.size == 0:
                raise ValueError("planted keys need a query on the sequence")
            t = int(qb[-1])
            if sp.index_dtype in ("e4m3", "mxfp8"):
                qdeq = torch.from_numpy(q_index[t]).view(torch.float8_e4m3fn).float().numpy()
                if sp.index_dtype == "mxfp8":
                    qdeq = qdeq * np.repeat(e8m0_value(q_index_scale[t]), MX_GROUP, axis=-1)
                else:
                    sc = q_index_scale[t]
                    qdeq = qdeq * (np.repeat(sc, sp.index_scale_group, axis=-1)
                                   if sp.index_scale_group else sc[:, None])
            elif sp.index_dtype == "bf16":
                qdeq = (q_index[t].astype(np.uint32) << 16).view(np.float32)
            else:
                qdeq = q_index[t]
            u = (np.maximum(w[t], 0.0)[:, None].astype(np.float64) * qdeq).sum(axis=0)
            u = (u / np.linalg.norm(u)).astype(np.float32)
        elif kind == "clusters":
            n_cl, span = int(sp.keys[1]), int(sp.keys[2])
            free = L - n_cl * span
            if free < 0:
                raise ValueError("clusters do not fit")
            gaps = np.sort(rng.integers(0, free + 1, size=n_cl))
            starts = gaps + span * np.arange(n_cl)
            centers = _normal(rng, (n_cl, d_I))
            clusters[b] = [(int(s), span) for s in starts]
        elif kind != "iid":
            raise ValueError(sp.keys)

        pt = page_table[b]
        for c0 in range(0, L, _CHUNK):
            c1 = min(L, c0 + _CHUNK)
            k = _normal(rng, (c1 - c0, d_I))
            if kind == "planted":
                sel = pos[(pos >= c0) & (pos < c1)] - c0
                k[sel] += np.float32(sigma) * u[None, :]
            elif kind == "clusters":
                for ci, (s0, n) in enumerate(clusters[b]):
                    a, e = max(s0, c0), min(s0 + n, c1)
                    if a < e:
                        k[a - c0:e - c0] = ((centers[ci][None, :] + k[a - c0:e - c0])
                                            / np.float32(math.sqrt(2.0)))
            dst = _phys_rows(pt, c0, c1, ps)
            if sp.index_dtype in ("e4m3", "mxfp8"):
                codes, sc = _quantize_index(k, sp.index_scale_group, sp.index_dtype == "mxfp8")
                k_index[dst] = codes
                k_index_scale[dst] = sc
            elif sp.index_dtype == "bf16":
                k_index[dst] = to_bf16_bits(k)
            else:
                k_index[dst] = k
    k_index = k_index.reshape(num_pages, ps, d_I)
    if k_index_scale is not None:
        k_index_scale = k_index_scale.reshape((num_pages, ps) + k_index_scale.shape[1:])

    # MLA latent cache
    D, dl, dr = sp.d_qk, sp.d_latent, sp.d_rope
    kv_rope = kv_scale = None
    if sp.kv_dtype == "f32":
        kv = np.full((rows, D), np.nan, dtype=np.float32)
    elif sp.kv_dtype == "bf16":
        kv = np.full((rows, D), BF16_NAN, dtype=np.uint16)
    elif sp.kv_dtype == "e4m3":
        if ps != 64:
            raise ValueError("the e4m3 cache keeps one scale per 64-token page")
        kv = np.full((rows, dl), E4M3_NAN, dtype=np.uint8)
        kv_rope = np.full((rows, dr), BF16_NAN, dtype=np.uint16)
        st, sd = sp.kv_tile
        if ps % st or dl % sd:
            raise ValueError("scale tiles must divide the page and the latent dims")
        kv_scale = np.full((num_pages, ps // st, dl // sd), np.nan, dtype=np.float32)
    else:
        raise ValueError(sp.kv_dtype)
    for b in range(sp.batch):
        L = int(lens[b])
        pt = page_table[b]
        for c0 in range(0, L, _CHUNK):
            c1 = min(L, c0 + _CHUNK)
            x = _normal(rng, (c1 - c0, D))
            dst = _phys_rows(pt, c0, c1, ps)
            if sp.kv_dtype == "f32":
                kv[dst] = x
            elif sp.kv_dtype == "bf16":
                kv[dst] = to_bf16_bits(x)
            else:
                # one scale per (st tokens x sd dims) tile of each page's
                # latent part; the chunk is a multiple of the page size, so
                # pages never straddle chunks
                lat = x[:, :dl]
                n = c1 - c0
                npg = (n + ps - 1) // ps
                pad = npg * ps - n
                lat_p = np.concatenate([lat, np.zeros((pad, dl), np.float32)]) if pad else lat
                tiles = np.abs(lat_p).reshape(npg, ps // st, st, dl // sd, sd)
                sc = amax_scale(tiles.max(axis=(2, 4)))            # [npg, ps/st, dl/sd]
                full = np.repeat(np.repeat(sc, st, axis=1), sd, axis=2).reshape(npg * ps, dl)
                codes = to_e4m3_codes(lat / full[:n])
                kv[dst] = codes
                kv_rope[dst] = to_bf16_bits(x[:, dl:])
                kv_scale[pt[c0 // ps: c0 // ps + npg]] = sc
    kv = kv.reshape(num_pages, ps, -1)
    if kv_rope is not None:
        kv_rope = kv_rope.reshape(num_pages, ps, dr)

    # attention queries (absorbed MLA: latent part + rope part)
    qx = _normal(rng, (n_q, sp.heads, D))
    q = qx if sp.q_dtype == "f32" else to_bf16_bits(qx)

    return Workload(spec=sp, seq_len=lens, page_table=page_table, num_pages=num_pages,
                    q_seq=q_seq, q_pos=q_pos, k_index=k_index, k_index_scale=k_index_scale,
                    q_index=q_index, q_index_scale=q_index_scale, w=w, kv=kv,
                    kv_rope=kv_rope, kv_scale=kv_scale, q=q, planted=planted,
                    clusters=clusters)


def permute_pages(wl: Workload, seed: int) -> Workload:
    """Same logical cache, different physical page placement."""
    rng = np.random.default_rng(seed)
    sigma = rng.permutation(wl.num_pages)
    inv = np.empty_like(sigma)
    inv[sigma] = np.arange(wl.num_pages)

    def move(a):
        if a is None:
            return None
        return np.ascontiguousarray(a[inv])

    pt = wl.page_table.copy()
    m = pt >= 0
    pt[m] = sigma[pt[m]]
    return dataclasses.replace(
        wl, page_table=pt, k_index=move(wl.k_index), k_index_scale=move(wl.k_index_scale),
        kv=move(wl.kv), kv_rope=move(wl.kv_rope), kv_scale=move(wl.kv_scale))


def shard_workload(wl: Workload, lo, hi) -> Workload:
    """The cache one rank of a context-parallel group holds: positions
    [lo[b], hi[b]) of every sequence (page-aligned lo), as local positions
    0 .. hi - lo - 1, in pools of its own holding only those pages (renumbered
    in the order of their logical positions) plus the unused poisoned pages;
    each decode query sits at its shard's last local position."""
    ps = wl.spec.page_size
    lo, hi = np.asarray(lo, np.int64), np.asarray(hi, np.int64)
    if np.any(lo % ps) or np.any(hi <= lo):
        raise ValueError("shards start on a page and hold at least one position")
    if wl.spec.queries[0] != "decode":
        raise ValueError("context-parallel shards serve decode queries")
    B = wl.seq_len.shape[0]
    n_pg = (hi - lo + ps - 1) // ps
    pages = [wl.page_table[b, lo[b] // ps: lo[b] // ps + n_pg[b]].astype(np.int64)
             for b in range(B)]
    keep = np.concatenate(pages + [np.setdiff1d(np.arange(wl.num_pages),
                                                wl.page_table[wl.page_table >= 0])])
    new_id = np.full(wl.num_pages, -1, np.int64)
    new_id[keep] = np.arange(keep.size)
    pt = np.full((B, int(n_pg.max())), -1, dtype=np.int32)
    for b in range(B):
        pt[b, :n_pg[b]] = new_id[pages[b]]

    def take(a):
        return None if a is None else np.ascontiguousarray(a[keep])

    lens = (hi - lo).astype(np.int32)
    return dataclasses.replace(
        wl, seq_len=lens, page_table=pt, num_pages=int(keep.size),
        q_pos=(lens[wl.q_seq] - 1).astype(np.int32),
        k_index=take(wl.k_index), k_index_scale=take(wl.k_index_scale), kv=take(wl.kv),
        kv_rope=take(wl.kv_rope), kv_scale=take(wl.kv_scale), planted={}, clusters={})


def subset_queries(wl: Workload, rows) -> Workload:
    """The same cache with only the queries ``rows`` (for sampled checks)."""
    rows = np.asarray(rows, dtype=np.int64)

    def take(a):
        return None if a is None else np.ascontiguousarray(a[rows])

    return dataclasses.replace(
        wl, q_seq=take(wl.q_seq), q_pos=take(wl.q_pos), q_index=take(wl.q_index),
        q_index_scale=take(wl.q_index_scale), w=take(wl.w), q=take(wl.q))


def stratified_rows(n: int, count: int) -> np.ndarray:
    """``count`` query rows spread evenly over ``0..n-1`` (first and last included)."""
    if count >= n:
        return np.arange(n)
    return np.unique(np.round(np.linspace(0, n - 1, count)).astype(np.int64))
