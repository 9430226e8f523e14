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
    if dtype in ("e4m3", "mxfp8"):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e4m3fn).double().numpy()
    raise ValueError(dtype)


def np_scales(dtype, a):
    """Scale values: fp32 as stored, or E8M0 bytes (MXFP8) through torch's decoder."""
    if dtype == "mxfp8":
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.float8_e8m0fnu).double().numpy()
    return np.asarray(a).astype(np.float64)


def np_rows(wl, b, positions):
    ps = wl.spec.page_size
    positions = np.asarray(positions, dtype=np.int64)
    return wl.page_table[b][positions // ps].astype(np.int64) * ps + positions % ps


def np_index_keys(wl, b, V):
    rows = np_rows(wl, b, np.arange(V))
    d = wl.spec.d_index
    k = np_values(wl.spec.index_dtype, wl.k_index.reshape(-1, d)[rows])
    if wl.k_index_scale is not None:
        per_row = wl.k_index_scale.reshape(wl.k_index.shape[0] * wl.k_index.shape[1], -1)[rows]
        per_row = np_scales(wl.spec.index_dtype, per_row)
        k = k * (np.repeat(per_row, d // per_row.shape[1], axis=1))
    return k


def np_scores(wl):
    out = np.full((wl.n_q, wl.max_visible), np.nan)
    for t in range(wl.n_q):
        V = int(wl.q_pos[t]) + 1
        k = np_index_keys(wl, int(wl.q_seq[t]), V)
        q = np_values(wl.spec.index_dtype, wl.q_index[t])
        if wl.q_index_scale is not None:
            qs = np_scales(wl.spec.index_dtype, wl.q_index_scale[t].reshape(wl.spec.h_index, -1))
            q = q * np.repeat(qs, wl.spec.d_index // qs.shape[1], axis=1)
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


def test_e8m0_decode_matches_torch_for_every_byte():
    """The MXFP8 scale bytes: b -> 2^(b - 127), 255 -> NaN (torch's float8_e8m0fnu)."""
    b = np.arange(256, dtype=np.uint8)
    ours = oracle.e8m0_decode(b).astype(np.float64)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref)) and np.isnan(ours[255])
    assert np.array_equal(ours[:255], ref[:255])
    assert ours[127] == 1.0 and ours[0] == 2.0 ** -127 and ours[254] == 2.0 ** 127


def test_mxfp8_inputs_follow_the_mx_scale_rule():
    """The input generator's MXFP8 groups: every scale is the power of two
    2^(floor(log2 amax) - 8), so the group's largest value lands in [256, 512)
    times the scale (saturated to 448), and every value is within half an e4m3
    step (or the saturation) of its input."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((40, 64)) * np.exp(rng.uniform(-20, 20, (40, 1)))).astype(np.float32)
    x[5, :32] = 0.0
    codes, b = W.quantize_mxfp8(x)
    sc = np_scales("mxfp8", b)
    g = x.reshape(40, 2, 32).astype(np.float64)
    amax = np.abs(g).max(axis=2)
    nz = amax > 0
    assert np.all(np.floor(np.log2(amax[nz])) - 8 == np.log2(sc[nz]))
    assert b[5, 0] == 127
    deq = np_values("e4m3", codes).reshape(40, 2, 32) * sc[..., None]
    top = np.abs(deq).max(axis=2)[nz] / sc[nz]
    assert np.all((top >= 256) & (top <= 448))
    err = np.abs(deq - g) / sc[..., None]
    assert np.all((err <= 16) | (np.abs(g) / sc[..., None] >= 448))


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

@pytest.mark.parametrize("index_dtype,group", [("f32", 0), ("bf16", 0), ("e4m3", 0),
                                               ("e4m3", 8), ("mxfp8", 0)])
def test_scores_match_brute_force(index_dtype, group):
    """group > 0: one e4m3 scale per `group` values of the query and key rows
    (the pages' group-wise index quantisation, here 8 of 16 dims); mxfp8: one
    E8M0 scale per 32 values (MXFP8, 64 dims)."""
    d = 64 if index_dtype == "mxfp8" else 16
    wl = W.make_workload(small_spec(index_dtype=index_dtype, index_scale_group=group,
                                    d_index=d))
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


# ------------------------------------------------------- input preparation ---
# Pins for the FP8 / bf16 encoders and the append scatter of the oracle.

def torch_e4m3(x):
    """torch's own fp32 -> e4m3fn conversion (round to nearest even)."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def e4m3_table():
    """All finite e4m3 codes and their values, from torch."""
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    return codes, vals


def test_e4m3_encoder_round_trips_every_finite_code():
    codes, vals = e4m3_table()
    got = oracle.e4m3_encode(vals)
    # -0 and +0 both encode by sign; every other value has exactly one code
    assert np.array_equal(got, codes)


def test_e4m3_encoder_matches_torch_including_ties():
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-12, np.log2(448.0), 20000)).astype(np.float32)
    x = mags * rng.choice([-1.0, 1.0], mags.size).astype(np.float32)
    _, vals = e4m3_table()
    v = np.unique(vals[vals > 0])
    mids = ((v[:-1].astype(np.float64) + v[1:]) / 2).astype(np.float32)  # exact in fp32
    x = np.concatenate([x, mids, -mids, np.float32(2.0 ** -10) * np.arange(1, 9,
                                                                            dtype=np.float32)])
    assert np.array_equal(oracle.e4m3_encode(x), torch_e4m3(x))


def test_e4m3_encoder_closed_forms():
    x = np.array([449, 464, 1e30, -1e30, 2 ** -10, 3 * 2 ** -10, 2 ** -9, 1.0625, 1.1875, 0.0,
                  -0.0, 240, 248, 256], dtype=np.float32)
    # 464 is the midpoint of 448 and (non-finite) 480: saturation keeps 448;
    # 2^-10 ties to 0 (even), 3*2^-10 to 2*2^-9, 1.0625 to 1.0, 1.1875 to 1.25;
    # 248 is the midpoint of 240 (mantissa 7, odd) and 256 (mantissa 0, even)
    want = [0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x02, 0x01, 0x38, 0x3A, 0x00, 0x80, 0x77, 0x78,
            0x78]
    assert oracle.e4m3_encode(x).tolist() == want


def test_bf16_encoder_matches_torch():
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2 ** 32, 50000, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]          # finite only
    ties = (rng.integers(0, 2 ** 16, 2000).astype(np.uint32) << 16) | 0x8000
    ties = ties[(ties & 0x7F800000) != 0x7F800000]
    x = np.concatenate([bits, ties]).view(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.to_bf16(x), want)


def test_group_quantisation_rule():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((300, 128)) * np.exp2(rng.uniform(-8, 8, (300, 1)))) \
        .astype(np.float32)
    x[7] = 0.0                                               # an all-zero group
    codes, scales = oracle.quantize_e4m3(x, 32)
    assert codes.shape == x.shape and scales.shape == (300, 4)
    g = x.reshape(300, 4, 32)
    amax = np.abs(g).max(axis=-1)
    want_scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(scales, want_scale)                # fp32 division, as numpy does it
    assert np.all(codes[7] == 0) and np.all(scales[7] == 1.0)
    # each code is torch's rounding of the fp32 quotient, so the largest
    # magnitude of every group lands on +-448
    q = (g / want_scale[..., None]).astype(np.float32)
    assert np.array_equal(codes.reshape(300, 4, 32), torch_e4m3(q))
    c = codes.reshape(300, 4, 32)
    top = np.take_along_axis(c, np.abs(g).argmax(axis=-1)[..., None], axis=-1)[..., 0]
    live = amax > 0
    assert np.all((top[live] & 0x7F) == 0x7E)
    # dequantised error within half an e4m3 step of the quotient
    _, vals = e4m3_table()
    deq = torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).float().numpy()
    step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -9))), -6) - 3)
    assert np.all(np.abs(deq - q) <= step / 2 + 1e-12)


def test_query_quantisation_agrees_with_the_input_generator():
    rng = np.random.default_rng(14)
    q = rng.standard_normal((9, 64, 128)).astype(np.float32)
    codes, scales = oracle.quantize_index_query(q)
    gen_codes, gen_scales = W.quantize_rows_e4m3(q)
    assert np.array_equal(codes, gen_codes) and np.array_equal(scales, gen_scales)


def _pools(rng, kv_dtype, P=6, ps=64, d_index=32, d_latent=64, d_rope=16, dims=16):
    pools = {"k_index": rng.integers(0, 255, (P, ps, d_index), dtype=np.uint8),
             "k_index_scale": rng.random((P, ps), dtype=np.float32),
             "kv_rope": None, "kv_scale": None}
    if kv_dtype == "e4m3":
        pools["kv"] = rng.integers(0, 255, (P, ps, d_latent), dtype=np.uint8)
        pools["kv_rope"] = rng.integers(0, 2 ** 15, (P, ps, d_rope), dtype=np.uint16)
        pools["kv_scale"] = rng.random((P, ps, d_latent // dims), dtype=np.float32)
    elif kv_dtype == "bf16":
        pools["kv"] = rng.integers(0, 2 ** 15, (P, ps, d_latent + d_rope), dtype=np.uint16)
    else:
        pools["kv"] = rng.random((P, ps, d_latent + d_rope), dtype=np.float32)
    return pools


@pytest.mark.parametrize("kv_dtype", ["e4m3", "bf16", "f32"])
def test_append_scatters_through_the_page_table(kv_dtype):
    rng = np.random.default_rng(15)
    P, ps, d_index, d_latent, d_rope, dims = 6, 64, 32, 64, 16, 16
    pools = _pools(rng, kv_dtype)
    table_a = np.array([[4, 1, -1], [0, 5, 9]], dtype=np.int32)   # 9: bad page id
    layout = {"page_table": table_a, "page_size": ps, "num_pages": P, "index_dtype": "e4m3",
              "kv_dtype": kv_dtype, "d_latent": d_latent, "kv_scale_dims": dims}
    seq = np.array([0, 0, 1, 1, 2, 0, -1, 1, 0])
    pos = np.array([3, 127, 64, 130, 0, 128, 0, 200, -5])
    k_new = rng.standard_normal((9, d_index)).astype(np.float32)
    kv_new = rng.standard_normal((9, d_latent + d_rope)).astype(np.float32)
    out, skipped = oracle.append_tokens(pools, layout, seq, pos, k_new, kv_new)
    # seq 0 pos 128 hits a -1 slot; seq 1 pos 130 hits page 9; pos 200 is past max_pages
    assert sorted(skipped) == [(3, "page"), (4, "position"), (5, "page"), (6, "position"),
                               (7, "position"), (8, "position")]
    written = {(4, 3): 0, (1, 63): 1, (5, 0): 2}                # (page, slot) -> token
    for name, a in pools.items():
        if a is None:
            continue
        changed = {(p, s) for p, s in zip(*np.nonzero(
            (out[name] != a).reshape(P, ps, -1).any(axis=-1)))}
        assert changed <= set(written), name
    for (page, slot), i in written.items():
        assert np.array_equal(out["k_index"][page, slot], torch_e4m3(
            k_new[i] / out["k_index_scale"][page, slot]))
        assert out["k_index_scale"][page, slot] == np.abs(k_new[i]).max() / np.float32(448)
        if kv_dtype == "e4m3":
            sc = out["kv_scale"][page, slot]
            lat = kv_new[i, :d_latent].reshape(-1, dims)
            assert np.array_equal(sc, np.abs(lat).max(axis=-1) / np.float32(448))
            assert np.array_equal(out["kv"][page, slot].reshape(-1, dims),
                                  torch_e4m3(lat / sc[:, None]))
            want_rope = torch.from_numpy(kv_new[i, d_latent:]).to(torch.bfloat16) \
                .view(torch.int16).numpy().view(np.uint16)
            assert np.array_equal(out["kv_rope"][page, slot], want_rope)
        elif kv_dtype == "bf16":
            want = torch.from_numpy(kv_new[i]).to(torch.bfloat16).view(torch.int16).numpy() \
                .view(np.uint16)
            assert np.array_equal(out["kv"][page, slot], want)
        else:
            assert np.array_equal(out["kv"][page, slot], kv_new[i])
    # the same tokens through a permuted table land at the same logical rows
    perm = np.array([2, 3, 0, 5, 1, 4])
    layout_b = dict(layout, page_table=np.where(table_a >= 0, perm[np.clip(table_a, 0, 5)],
                                                table_a).astype(np.int32))
    layout_b["page_table"][1, 2] = 9
    pools_b = {k: None if v is None else v[np.argsort(perm)] for k, v in pools.items()}
    out_b, skipped_b = oracle.append_tokens(pools_b, layout_b, seq, pos, k_new, kv_new)
    assert skipped_b == skipped
    for name in pools:
        if pools[name] is not None:
            assert np.array_equal(out_b[name][perm], out[name])
