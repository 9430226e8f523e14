"""Parity rules shared by the GPU tests (and unit-tested on the CPU).

Top-K: the GPU index set must equal the oracle's, except that a position may be
swapped for another only when both oracle scores lie within the tie window of
the oracle's K-th score: ``|I[s] - s_K| <= max(1e-3 * |s_K|, 1e-6 * max|I|)``.
Attention (recomputed by the oracle on the GPU's own index set): max-abs error
<= 2e-2 and mean-rel error ``sum|g - o| / sum|o|`` <= 5e-3 for a bf16 cache,
max-abs <= 6e-2 for the FP8 latent cache.
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-3
TIE_FLOOR = 1e-6
ATTN_MAX_ABS = {"f32": 2e-2, "bf16": 2e-2, "e4m3": 6e-2}
ATTN_MEAN_REL = {"f32": 5e-3, "bf16": 5e-3, "e4m3": None}


class ParityError(AssertionError):
    pass


def check_topk(gpu_idx: np.ndarray, oracle_scores: np.ndarray, valid: np.ndarray, K: int,
               oracle_idx: np.ndarray | None = None) -> dict:
    """Validate ``gpu_idx`` [n_q, K] against oracle scores [n_q, >= max V]."""
    gpu_idx = np.asarray(gpu_idx)
    n_q = gpu_idx.shape[0]
    swaps = 0
    worst = 0.0
    for t in range(n_q):
        V = int(valid[t])
        n = min(K, V)
        row = gpu_idx[t]
        sel, pad = row[:n], row[n:]
        if np.any(pad != -1):
            raise ParityError(f"query {t}: padding is not -1")
        if np.any(sel < 0) or np.any(sel >= V):
            raise ParityError(f"query {t}: index outside [0, {V})")
        if np.any(np.diff(sel) <= 0):
            raise ParityError(f"query {t}: indices not strictly ascending")
        sc = oracle_scores[t, :V]
        if oracle_idx is not None:
            ref = oracle_idx[t, :n]
        else:
            order = np.lexsort((np.arange(V), -sc))
            ref = np.sort(order[:n])
        if np.array_equal(sel, ref):
            continue
        s_k = sc[ref].min()
        tol = max(TIE_REL * abs(s_k), TIE_FLOOR * float(np.abs(sc).max()))
        diff = np.setxor1d(sel, ref)
        dev = np.abs(sc[diff] - s_k)
        worst = max(worst, float(dev.max() / max(tol, 1e-300)))
        if np.any(dev > tol):
            bad = diff[dev > tol][:5]
            raise ParityError(
                f"query {t}: {diff.size} differing positions, e.g. {bad.tolist()} with "
                f"scores {sc[bad].tolist()} vs K-th score {s_k} (tol {tol})")
        swaps += diff.size // 2
    return {"swaps": swaps, "worst_window_fraction": worst}


def attention_errors(gpu_out: np.ndarray, ref_out: np.ndarray) -> dict:
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ref_out, dtype=np.float64)
    if not np.all(np.isfinite(g)):
        return {"max_abs": float("inf"), "mean_rel": float("inf")}
    d = np.abs(g - o)
    return {"max_abs": float(d.max()) if d.size else 0.0,
            "mean_rel": float(d.sum() / max(np.abs(o).sum(), 1e-300))}


def check_attention(gpu_out, ref_out, kv_dtype: str) -> dict:
    e = attention_errors(gpu_out, ref_out)
    if not e["max_abs"] <= ATTN_MAX_ABS[kv_dtype]:
        raise ParityError(f"attention max-abs {e['max_abs']} > {ATTN_MAX_ABS[kv_dtype]}")
    lim = ATTN_MEAN_REL[kv_dtype]
    if lim is not None and not e["mean_rel"] <= lim:
        raise ParityError(f"attention mean-rel {e['mean_rel']} > {lim}")
    return e


def check_lse(gpu_lse, ref_lse, tol: float = 1e-2) -> float:
    d = float(np.max(np.abs(np.asarray(gpu_lse, np.float64) - ref_lse)))
    if not d <= tol:
        raise ParityError(f"lse max-abs {d} > {tol}")
    return d
