"""fp64 CPU oracle for indexed sparse attention (ctypes wrapper over sa_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it; the library under
``indexed_sparse_attention_lightning_b200`` never imports it.  It shares no code
with the CUDA path.  Inputs are plain numpy arrays (any object with the
attributes of a workload works); all arithmetic is in ``sa_oracle.c``.

Pins: every function here is checked in ``tests/test_oracle.py`` against
something other than itself (numpy brute force on tiny inputs, closed forms,
invariants, a hand-worked example under ``tests/golden/``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16, E4M3 = 0, 1, 2
_DT = {"f32": F32, "bf16": BF16, "e4m3": E4M3}
_ERR = {-1: "bad argument", -2: "page id out of range", -3: "index outside visible range",
        -4: "NaN encountered", -5: "out of memory"}

_lib = None


def build(force: bool = False) -> str:
    """Compile sa_oracle.c with gcc (plain C11, -O2)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_decode.argtypes = [ctypes.c_int, P, P, I64]
        lib.oracle_decode.restype = None
        lib.oracle_index_scores.argtypes = [I32, P, P, I32, I32, I32, I32, P, P, P, I32, P, P,
                                            P, I32, I32, I32, P, I64, ctypes.c_int]
        lib.oracle_index_scores.restype = ctypes.c_int
        lib.oracle_topk.argtypes = [I32, P, I64, P, I32, P]
        lib.oracle_topk.restype = ctypes.c_int
        lib.oracle_sparse_attn.argtypes = [I32, P, P, I32, I32, I32, I32, P, D, I32, P, P, P,
                                           I32, I32, P, I32, I32, I32, P, I32, P, P,
                                           ctypes.c_int]
        lib.oracle_sparse_attn.restype = ctypes.c_int
        lib.oracle_quantize_e4m3.argtypes = [I64, I32, P, P, P]
        lib.oracle_quantize_e4m3.restype = ctypes.c_int
        lib.oracle_e4m3_encode.argtypes = [I64, P, P]
        lib.oracle_e4m3_encode.restype = ctypes.c_int
        lib.oracle_to_bf16.argtypes = [I64, P, P]
        lib.oracle_to_bf16.restype = ctypes.c_int
        lib.oracle_e8m0_decode.argtypes = [I64, P, P]
        lib.oracle_e8m0_decode.restype = ctypes.c_int
        _lib = lib
    return _lib


def threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: {_ERR.get(rc, rc)}")


def decode(dtype: str, codes: np.ndarray) -> np.ndarray:
    """Widen stored values (f32 / bf16 bits / e4m3 codes) to float64."""
    src = np.ascontiguousarray(codes)
    out = np.empty(src.shape, dtype=np.float64)
    _load().oracle_decode(_DT[dtype], _ptr(src), _ptr(out), src.size)
    return out


MX_GROUP = 32  # values per E8M0 scale in the MXFP8 format


def e8m0_decode(b: np.ndarray) -> np.ndarray:
    """E8M0 scale bytes -> fp32 values 2^(b - 127) (255 -> NaN), exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, dtype=np.float32)
    _check(_load().oracle_e8m0_decode(b.size, _ptr(b), _ptr(out)), "e8m0_decode")
    return out


def _index_dtype(wl):
    return wl.spec.index_dtype


def index_scores(wl, nthreads: int | None = None) -> np.ndarray:
    """I[t, s] for s < V_t (float64 [n_q, max V]; NaN past each V_t).  MXFP8
    inputs (e4m3 codes, one E8M0 byte per 32 values) are scored as e4m3 codes
    with those group scales decoded to fp32 (exact: powers of two)."""
    n_q = wl.n_q
    ld = max(1, wl.max_visible)
    scores = np.full((n_q, ld), np.nan, dtype=np.float64)
    mx = _index_dtype(wl) == "mxfp8"
    dt = _DT["e4m3" if mx else _index_dtype(wl)]
    group = MX_GROUP if mx else getattr(wl.spec, "index_scale_group", 0)
    qi = np.ascontiguousarray(wl.q_index)
    ki = np.ascontiguousarray(wl.k_index)
    if mx:
        qs, ks = e8m0_decode(wl.q_index_scale), e8m0_decode(wl.k_index_scale)
    else:
        qs, ks = _c(wl.q_index_scale, np.float32), _c(wl.k_index_scale, np.float32)
    w = _c(wl.w, np.float32)
    q_seq, q_pos = _c(wl.q_seq, np.int32), _c(wl.q_pos, np.int32)
    pt = _c(wl.page_table, np.int32)
    rc = _load().oracle_index_scores(
        n_q, _ptr(q_seq), _ptr(q_pos), wl.spec.h_index, wl.spec.d_index, group,
        dt, _ptr(qi), _ptr(qs), _ptr(w), dt, _ptr(ki), _ptr(ks),
        _ptr(pt), pt.shape[1], wl.spec.page_size, wl.num_pages,
        _ptr(scores), ld, nthreads or threads())
    _check(rc, "index_scores")
    return scores


def topk(scores: np.ndarray, valid: np.ndarray, K: int) -> np.ndarray:
    """Ascending top-K positions per row (int32 [n_q, K], -1 padded)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    v = np.ascontiguousarray(valid, dtype=np.int32)
    idx = np.empty((s.shape[0], K), dtype=np.int32)
    rc = _load().oracle_topk(s.shape[0], _ptr(s), s.shape[1], _ptr(v), K, _ptr(idx))
    _check(rc, "topk")
    return idx


def sparse_attn(wl, idx: np.ndarray, nthreads: int | None = None):
    """(out float64 [n_q, heads, d_latent], lse float64 [n_q, heads]) on rows ``idx``."""
    sp = wl.spec
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n_q, K = idx.shape
    out = np.empty((n_q, sp.heads, sp.d_latent), dtype=np.float64)
    lse = np.empty((n_q, sp.heads), dtype=np.float64)
    q = np.ascontiguousarray(wl.q)
    kv = np.ascontiguousarray(wl.kv)
    rope = None if wl.kv_rope is None else np.ascontiguousarray(wl.kv_rope)
    ksc = _c(wl.kv_scale, np.float32)
    q_seq, q_pos = _c(wl.q_seq, np.int32), _c(wl.q_pos, np.int32)
    pt = _c(wl.page_table, np.int32)
    rc = _load().oracle_sparse_attn(
        n_q, _ptr(q_seq), _ptr(q_pos), sp.heads, sp.d_latent, sp.d_rope,
        _DT[sp.q_dtype], _ptr(q), sp.softmax_scale, _DT[sp.kv_dtype], _ptr(kv), _ptr(rope),
        _ptr(ksc), sp.kv_tile[0], sp.kv_tile[1],
        _ptr(pt), pt.shape[1], sp.page_size, wl.num_pages, _ptr(idx), K,
        _ptr(out), _ptr(lse), nthreads or threads())
    _check(rc, "sparse_attn")
    return out, lse


# ---------------------------------------------------------------------------
# Input preparation ("Optimizing Next-Gen LLM Inference", §3.2 and the §4
# table; "Inference Acceleration for New Large Model Architectures", §3.3 and
# §4.1-4.2).  The arithmetic (scale, quotient, rounding) is in sa_oracle.c;
# this part only reshapes and scatters.
# ---------------------------------------------------------------------------

def widen(dtype: str, a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) or fp32 values -> fp32 values, exactly."""
    if dtype == "bf16":
        return (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(a, dtype=np.float32)


def quantize_e4m3(x: np.ndarray, group: int):
    """Dynamic FP8 quantisation of the last axis in groups of ``group`` values:
    (codes uint8, same shape; scales f32 [..., last / group])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.shape[-1] % group:
        raise ValueError("the last axis must be a multiple of the group")
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (x.shape[-1] // group,), dtype=np.float32)
    rc = _load().oracle_quantize_e4m3(x.size // group, group, _ptr(x), _ptr(codes), _ptr(scales))
    _check(rc, "quantize_e4m3")
    return codes, scales


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 values -> e4m3 codes (round to nearest even, saturating), no scale."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.empty(x.shape, dtype=np.uint8)
    _check(_load().oracle_e4m3_encode(x.size, _ptr(x), _ptr(codes)), "e4m3_encode")
    return codes


def to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = np.empty(x.shape, dtype=np.uint16)
    _check(_load().oracle_to_bf16(x.size, _ptr(x), _ptr(bits)), "to_bf16")
    return bits


def quantize_index_query(q: np.ndarray):
    """Indexer query [n_q, h, d] (fp32 values) -> e4m3 codes + one scale per
    (token, head): the form the FP8 indexer consumes."""
    codes, scales = quantize_e4m3(q, q.shape[-1])
    return codes, scales[..., 0]


def append_tokens(pools: dict, layout: dict, seq, pos, k_new=None, kv_new=None):
    """Write new tokens into copies of the paged pools.

    pools: ``k_index``, ``k_index_scale``, ``kv``, ``kv_rope``, ``kv_scale`` (numpy
    arrays shaped as the cache stores them; absent entries are None).
    layout: ``page_table`` [batch, max_pages], ``page_size``, ``num_pages``,
    ``index_dtype`` ("e4m3"/"bf16"/"f32"), ``kv_dtype`` ("e4m3"/"bf16"/"f32"), ``d_latent``,
    ``kv_scale_dims`` (latent dims per scale; one token per scale).
    k_new [n, d_index], kv_new [n, d_latent + d_rope]: fp32 values.
    Token i goes to physical row page_table[seq, pos // page_size] * page_size +
    pos % page_size; a token whose sequence, position or page id is out of range
    is skipped.  Returns (new pools, list of (token, "position" | "page") skips)."""
    out = {k: (None if v is None else v.copy()) for k, v in pools.items()}
    pt = layout["page_table"]
    ps, n_pages = layout["page_size"], layout["num_pages"]
    dl = layout["d_latent"]
    skipped = []
    for i, (b, p) in enumerate(zip(np.asarray(seq).tolist(), np.asarray(pos).tolist())):
        if not (0 <= b < pt.shape[0]) or p < 0 or p // ps >= pt.shape[1]:
            skipped.append((i, "position"))
            continue
        page = int(pt[b, p // ps])
        if not (0 <= page < n_pages):
            skipped.append((i, "page"))
            continue
        slot = p % ps
        if k_new is not None:
            if layout["index_dtype"] == "e4m3":
                codes, sc = quantize_e4m3(k_new[i], k_new.shape[-1])
                out["k_index"][page, slot] = codes
                out["k_index_scale"][page, slot] = sc[0]
            elif layout["index_dtype"] == "bf16":
                out["k_index"][page, slot] = to_bf16(k_new[i])
            else:
                out["k_index"][page, slot] = k_new[i]
        if kv_new is not None:
            row = np.asarray(kv_new[i], dtype=np.float32)
            if layout["kv_dtype"] == "e4m3":
                codes, sc = quantize_e4m3(row[:dl], layout["kv_scale_dims"])
                out["kv"][page, slot] = codes
                out["kv_scale"][page, slot] = sc
                out["kv_rope"][page, slot] = to_bf16(row[dl:])
            elif layout["kv_dtype"] == "bf16":
                out["kv"][page, slot] = to_bf16(row)
            else:
                out["kv"][page, slot] = row
    return out, skipped


def run(wl, nthreads: int | None = None) -> dict:
    """The whole path: scores -> top-K -> sparse attention."""
    scores = index_scores(wl, nthreads)
    idx = topk(scores, wl.visible, wl.spec.top_k)
    out, lse = sparse_attn(wl, idx, nthreads)
    return {"scores": scores, "idx": idx, "out": out, "lse": lse}


if __name__ == "__main__":  # pragma: no cover
    build(force="--force" in sys.argv)
    print(_LIB)
