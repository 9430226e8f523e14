"""Pins for the fp64 oracle, independent of the oracle's own code.

Each test checks the oracle against something other than itself: torch's own
fp8/bf16 conversions, numpy brute force on tiny inputs (its own page gather,
einsum, lexsort, dense softmax), closed forms, invariants, planted structure
and the hand-worked example in ``tests/golden/``.  A plausible slip in the
oracle -- a dropped ReLU or scale, a wrong sign, a swapped operand, a wrong page
lookup, a wrong tie rule -- fails at least one of them.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_lightning_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


# ---------------------------------------------------------------- helpers ---

def np_values(dtype, a):
    """Independent widening: torch for e4m3, bit shifts for bf16."""
    a = np.asarray(a)
    if dtype == "f32":
        return a.astype(np.float64)
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "e4m3":
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).double().numpy()
    raise ValueError(dtype)


def np_rows(wl, b, positions):
    ps = wl.spec.page_size
    positions = np.asarray(positions, dtype=np.int64)
    return wl.page_table[b][positions // ps].astype(np.int64) * ps + positions % ps


def np_index_keys(wl, b, V):
    rows = np_rows(wl, b, np.arange(V))
    k = np_values(wl.spec.index_dtype, wl.k_index.reshape(-1, wl.spec.d_index)[rows])
    if wl.k_index_scale is not None:
        k = k * wl.k_index_scale.reshape(-1)[rows][:, None].astype(np.float64)
    return k


def np_scores(wl):
    out = np.full((wl.n_q, wl.max_visible), np.nan)
    for t in range(wl.n_q):
        V = int(wl.q_pos[t]) + 1
        k = np_index_keys(wl, int(wl.q_seq[t]), V)
        q = np_values(wl.spec.index_dtype, wl.q_index[t])
        if wl.q_index_scale is not None:
            q = q * wl.q_index_scale[t][:, None].astype(np.float64)
        dots = np.einsum("sd,jd->sj", k, q)
        out[t, :V] = np.maximum(dots, 0.0) @ wl.w[t].astype(np.float64)
    return out


def np_latent_rows(wl, b, positions):
    sp = wl.spec
    rows = np_rows(wl, b, positions)
    if sp.kv_dtype == "e4m3":
        lat = np_values("e4m3", wl.kv.reshape(-1, sp.d_latent)[rows])
        # scale tile of (token, dim): (page, token // tile tokens, dim // tile dims)
        st, sd = sp.kv_tile
        sc = wl.kv_scale.reshape(wl.num_pages, sp.page_size // st, sp.d_latent // sd)
        per_row = sc[rows // sp.page_size, (rows % sp.page_size) // st]   # [n, d_latent / sd]
        lat = lat * np.repeat(per_row, sd, axis=1).astype(np.float64)
        rope = np_values("bf16", wl.kv_rope.reshape(-1, sp.d_rope)[rows])
        return np.concatenate([lat, rope], axis=1)
    return np_values(sp.kv_dtype, wl.kv.reshape(-1, sp.d_qk)[rows])


def np_dense_attention(wl):
    """Dense causal softmax attention over every visible row."""
    sp = wl.spec
    out = np.empty((wl.n_q, sp.heads, sp.d_latent))
    lse = np.empty((wl.n_q, sp.heads))
    for t in range(wl.n_q):
        V = int(wl.q_pos[t]) + 1
        rows = np_latent_rows(wl, int(wl.q_seq[t]), np.arange(V))
        q = np_values(sp.q_dtype, wl.q[t])
        z = sp.softmax_scale * (q @ rows.T)
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        out[t] = (e / e.sum(axis=1, keepdims=True)) @ rows[:, :sp.d_latent]
        lse[t] = m[:, 0] + np.log(e.sum(axis=1))
    return out, lse


def small_spec(**kw):
    base = dict(name="small", seed=11, batch=3, seq_len=("uniform", 150, 400),
                h_index=4, d_index=16, index_dtype="e4m3", top_k=48, heads=3,
                d_latent=24, d_rope=8, kv_dtype="bf16", q_dtype="bf16", page_size=16)
    base.update(kw)
    return W.WorkloadSpec(**base)


# ------------------------------------------------------- storage formats ---

def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode("e4m3", codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=4096, dtype=np.uint16)
    bits[:4] = [0x0000, 0x8000, 0x3F80, 0xC040]
    ours = oracle.decode("bf16", bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert list(ours[:4]) == [0.0, -0.0, 1.0, -3.0]


# --------------------------------------------------------- indexer score ---

@pytest.mark.parametrize("index_dtype", ["f32", "e4m3"])
def test_scores_match_brute_force(index_dtype):
    wl = W.make_workload(small_spec(index_dtype=index_dtype))
    got = oracle.index_scores(wl)
    ref = np_scores(wl)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_allclose(got[ok], ref[ok], rtol=1e-12, atol=1e-12)


def test_scores_closed_form_one_hot():
    """q_I[j] = e_j and k_I[s] = c_s e_{h(s)} give I[s] = w[h(s)] * c_s exactly."""
    H, d, L = 4, 8, 40
    sp = small_spec(batch=1, seq_len=("fixed", L), h_index=H, d_index=d, index_dtype="f32",
                    page_size=8, paging="permuted")
    wl = W.make_workload(sp)
    w = np.array([[0.75, -0.5, 1.25, 2.0]], dtype=np.float32)
    q = np.zeros((1, H, d), np.float32)
    q[0, np.arange(H), np.arange(H)] = 1.0
    c = (np.arange(L, dtype=np.float32) + 1.0) / 8.0
    head = np.arange(L) % H
    keys = np.zeros((L, d), np.float32)
    keys[np.arange(L), head] = c
    keys[::5, head[::5]] *= -1.0                 # negative dots are cut by the ReLU
    flat = wl.k_index.reshape(-1, d)
    flat[np_rows(wl, 0, np.arange(L))] = keys
    wl = dataclasses.replace(wl, q_index=q, w=w)
    got = oracle.index_scores(wl)[0, :L]
    expect = np.where(np.arange(L) % 5 == 0, 0.0, w[0, head].astype(np.float64) * c)
    assert np.array_equal(got, expect)


# ------------------------------------------------------------------ top-K ---

def test_topk_matches_lexsort_with_many_ties():
    rng = np.random.default_rng(3)
    n_q, L, K = 6, 500, 37
    scores = np.round(rng.standard_normal((n_q, L)), 1)  # heavy ties
    valid = np.array([500, 499, 37, 36, 1, 250], np.int32)
    got = oracle.topk(scores, valid, K)
    for t in range(n_q):
        V = valid[t]
        order = np.lexsort((np.arange(V), -scores[t, :V]))
        ref = np.sort(order[:min(K, V)])
        assert np.array_equal(got[t, :len(ref)], ref)
        assert np.all(got[t, len(ref):] == -1)


def test_topk_constant_scores_take_lowest_positions():
    scores = np.zeros((2, 300))
    got = oracle.topk(scores, np.array([300, 10], np.int32), 64)
    assert np.array_equal(got[0], np.arange(64))
    assert np.array_equal(got[1, :10], np.arange(10)) and np.all(got[1, 10:] == -1)


def test_planted_keys_are_the_top_k():
    """Keys pushed +20 sd along the query direction are exactly the selected set."""
    sp = small_spec(batch=2, seq_len=("fixed", 512), index_dtype="f32", h_index=4, d_index=16,
                    keys=("planted", 0.0625, 20.0), top_k=32)
    wl = W.make_workload(sp)
    # every head looks along the same direction, all head weights positive
    q = np.repeat(wl.q_index[:, :1, :], sp.h_index, axis=1)
    w = np.abs(wl.w) + 0.1
    wl2 = dataclasses.replace(wl, q_index=q, w=w.astype(np.float32))
    # re-plant along this query's direction
    for b in range(sp.batch):
        u = q[b, 0] / np.linalg.norm(q[b, 0])
        rows = np_rows(wl2, b, wl.planted[b])
        base = wl2.k_index.reshape(-1, sp.d_index)
        base[rows] = base[rows] - (base[rows] @ u)[:, None] * u[None, :] + 20.0 * u[None, :]
    res = oracle.topk(oracle.index_scores(wl2), wl2.visible, sp.top_k)
    for b in range(sp.batch):
        assert np.array_equal(res[b], wl.planted[b])


# ------------------------------------------------------------ attention ---

@pytest.mark.parametrize("kv_dtype,q_dtype", [("f32", "f32"), ("bf16", "bf16")])
def test_attention_equals_dense_when_k_covers_context(kv_dtype, q_dtype):
    sp = small_spec(kv_dtype=kv_dtype, q_dtype=q_dtype, top_k=512)
    wl = W.make_workload(sp)
    idx = oracle.topk(oracle.index_scores(wl), wl.visible, sp.top_k)
    out, lse = oracle.sparse_attn(wl, idx)
    ref_out, ref_lse = np_dense_attention(wl)
    np.testing.assert_allclose(out, ref_out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("tile", [(64, 32), (1, 16), (8, 8), (16, 32)])
def test_attention_fp8_latent_equals_dense(tile):
    """Every scale tile shape: the oracle's dequantisation (C, its own tile
    lookup) against numpy's restatement of the tile layout."""
    sp = small_spec(kv_dtype="e4m3", page_size=64, seq_len=("uniform", 130, 260), top_k=300,
                    d_latent=32, d_rope=8, kv_scale_tile=tile)
    wl = W.make_workload(sp)
    idx = oracle.topk(oracle.index_scores(wl), wl.visible, sp.top_k)
    out, lse = oracle.sparse_attn(wl, idx)
    ref_out, ref_lse = np_dense_attention(wl)
    np.testing.assert_allclose(out, ref_out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_single_row_returns_that_latent():
    wl = W.make_workload(small_spec())
    idx = np.full((wl.n_q, 4), -1, np.int32)
    idx[:, 1] = np.minimum(wl.q_pos, 17)
    out, lse = oracle.sparse_attn(wl, idx)
    sp = wl.spec
    for t in range(wl.n_q):
        row = np_latent_rows(wl, int(wl.q_seq[t]), [idx[t, 1]])[0]
        assert np.array_equal(out[t], np.broadcast_to(row[:sp.d_latent], out[t].shape))
        z = sp.softmax_scale * (np_values(sp.q_dtype, wl.q[t]) @ row)
        np.testing.assert_allclose(lse[t], z, rtol=1e-13, atol=1e-13)


def test_attention_zero_query_is_mean_of_rows():
    wl = W.make_workload(small_spec())
    wl = dataclasses.replace(wl, q=np.zeros_like(wl.q))
    idx = oracle.topk(oracle.index_scores(wl), wl.visible, wl.spec.top_k)
    out, lse = oracle.sparse_attn(wl, idx)
    for t in range(wl.n_q):
        sel = idx[t][idx[t] >= 0]
        rows = np_latent_rows(wl, int(wl.q_seq[t]), sel)[:, :wl.spec.d_latent]
        np.testing.assert_allclose(out[t], np.broadcast_to(rows.mean(axis=0), out[t].shape),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[t], math.log(sel.size), rtol=1e-14)


def test_attention_softmax_shift_invariance():
    """A constant rope column shifts every logit equally: output unchanged."""
    sp = small_spec(kv_dtype="f32", q_dtype="f32")
    wl = W.make_workload(sp)
    kv = wl.kv.copy()
    kv[..., -1] = 1.0
    q0 = wl.q.copy()
    q0[..., -1] = 0.25
    wl = dataclasses.replace(wl, kv=kv, q=q0)
    idx = oracle.topk(oracle.index_scores(wl), wl.visible, sp.top_k)
    out0, lse0 = oracle.sparse_attn(wl, idx)
    c = 3.5
    q1 = q0.copy()
    q1[..., -1] = 0.25 + c                      # exact in fp32
    out1, lse1 = oracle.sparse_attn(dataclasses.replace(wl, q=q1), idx)
    np.testing.assert_allclose(out1, out0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse1 - lse0, c * sp.softmax_scale, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------- layout ---

@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_page_permutation_leaves_everything_bit_identical(kv_dtype):
    sp = small_spec(kv_dtype=kv_dtype, page_size=64 if kv_dtype == "e4m3" else 16)
    wl = W.make_workload(sp)
    a = oracle.run(wl)
    b = oracle.run(W.permute_pages(wl, seed=99))
    for k in ("scores", "idx", "out", "lse"):
        assert np.array_equal(a[k], b[k], equal_nan=True), k


def test_poisoned_slots_are_never_read():
    """Slots past the end hold NaN; a correct oracle never touches them."""
    wl = W.make_workload(small_spec(seq_len=("uniform", 17, 200)))
    res = oracle.run(wl)
    assert np.all(np.isfinite(res["out"])) and np.all(np.isfinite(res["lse"]))
    # reading past the end is detected
    bad = dataclasses.replace(wl, q_pos=wl.q_pos + 1)
    with pytest.raises(ValueError):
        oracle.index_scores(bad)


def test_bad_page_id_is_reported():
    wl = W.make_workload(small_spec())
    pt = wl.page_table.copy()
    pt[0, 0] = wl.num_pages + 5
    with pytest.raises(ValueError, match="page"):
        oracle.index_scores(dataclasses.replace(wl, page_table=pt))


def test_index_outside_visible_range_is_reported():
    wl = W.make_workload(small_spec())
    idx = np.full((wl.n_q, 4), -1, np.int32)
    idx[0, 0] = wl.q_pos[0] + 1
    with pytest.raises(ValueError, match="visible"):
        oracle.sparse_attn(wl, idx)


# --------------------------------------------------------------- golden ---

def _golden_workload(g_ix, g_at):
    ps = g_ix["page_size"]
    pt = np.array(g_ix["page_table"], np.int32)
    keys = np.array(g_ix["keys_logical"], np.float32)
    L = keys.shape[0]
    k_index = np.zeros((pt.shape[1], ps, keys.shape[1]), np.float32)
    rows = [int(pt[0, s // ps]) * ps + s % ps for s in range(L)]
    k_index.reshape(-1, keys.shape[1])[rows] = keys
    dl, dr = g_at["d_latent"], g_at["d_rope"]
    rl = np.array(g_at["rows_logical"], np.float32)
    kv = np.zeros((pt.shape[1], ps, dl + dr), np.float32)
    for s in range(rl.shape[0]):
        kv.reshape(-1, dl + dr)[int(pt[0, s // ps]) * ps + s % ps] = rl[s]
    sp = W.WorkloadSpec(name="golden", seed=0, batch=1, seq_len=("fixed", L),
                        h_index=len(g_ix["w"]), d_index=keys.shape[1], index_dtype="f32",
                        top_k=2, heads=1, d_latent=dl, d_rope=dr, kv_dtype="f32",
                        q_dtype="f32", page_size=ps, sm_scale=g_at["sm_scale"])
    return W.Workload(
        spec=sp, seq_len=np.array([L], np.int32), page_table=pt, num_pages=pt.shape[1],
        q_seq=np.zeros(1, np.int32), q_pos=np.array([L - 1], np.int32), k_index=k_index,
        k_index_scale=None, q_index=np.array([g_ix["q_index"]], np.float32),
        q_index_scale=None, w=np.array([g_ix["w"]], np.float32), kv=kv, kv_rope=None,
        kv_scale=None, q=np.array([[g_at["q"]]], np.float32))


def test_golden_worked_example():
    g = json.load(open(GOLDEN))
    wl = _golden_workload(g["indexer"], g["attention"])
    scores = oracle.index_scores(wl)
    assert list(scores[0]) == g["indexer"]["scores"]
    for K, key in ((2, "top2"), (3, "top3"), (8, "top8")):
        assert oracle.topk(scores, wl.visible, K)[0].tolist() == g["indexer"][key]
    for case in g["attention"]["cases"]:
        out, lse = oracle.sparse_attn(wl, np.array([case["idx"]], np.int32))
        np.testing.assert_allclose(out[0, 0], case["out"], rtol=1e-15, atol=1e-16)
        np.testing.assert_allclose(lse[0, 0], case["lse"], rtol=1e-15)


# ------------------------------------------------------- parity checker ---

def test_parity_checker_accepts_tie_swaps_and_rejects_real_errors():
    from tests.parity import ParityError, check_topk
    scores = np.array([[5.0, 1.0, 3.0, 3.0000001, 0.5, 2.0]])
    valid = np.array([6])
    ref = oracle.topk(scores, valid, 3)          # [0, 2, 3]
    assert ref[0].tolist() == [0, 2, 3]
    check_topk(ref, scores, valid, 3)
    check_topk(np.array([[0, 2, 3]]), scores, valid, 3)
    # swapping 2 for 5 is outside the window (3 vs 2)
    with pytest.raises(ParityError):
        check_topk(np.array([[0, 3, 5]]), scores, valid, 3)
    # not ascending / duplicates / bad padding
    with pytest.raises(ParityError):
        check_topk(np.array([[2, 0, 3]]), scores, valid, 3)
    with pytest.raises(ParityError):
        check_topk(np.array([[0, 0, 3]]), scores, valid, 3)
    # a near-tie swap inside the window is accepted
    scores2 = np.array([[5.0, 1.0, 3.0, 3.0000001, 0.5, 3.0000002]])
    r = check_topk(np.array([[0, 2, 5]]), scores2, valid, 3)
    assert r["swaps"] == 1
