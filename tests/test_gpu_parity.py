"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

For every configuration the fused ``sa_decode`` runs on all queries -- the
launch that ``bench.py`` times -- and the oracle checks a stratified sample of
queries (all of them where it finishes in seconds):

* top-K: bit-exact index sets, except swaps among positions whose oracle score
  lies within ``max(1e-3 |s_K|, 1e-6 max|I|)`` of the oracle's K-th score;
* attention, recomputed by the oracle on the GPU's own index set: max-abs
  <= 2e-2 and mean-rel <= 5e-3 (bf16 / fp32 cache), max-abs <= 6e-2 (e4m3 latent);
* lse within 1e-2 absolute.

The unfused chain must agree with the fused path exactly, ``sa_topk`` must be
bit-exact against the oracle's selection on the same fp32 scores, and device
data errors must surface through the status word without a fault.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_lightning_b200 import _abi, api
from indexed_sparse_attention_lightning_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

# configuration -> number of oracle-checked queries (None = all).  Every decode
# query is checked; the prefill chunk checks 256 of its 4096 queries, spread
# evenly over the chunk (first and last included), so that every stretch of
# the persistent kernels' work lists is covered.
SAMPLES = {
    "tiny_decode_b1_1k_fp32": None,
    "decode_b8_8k": None,
    "decode_b64_16k_32k_planted": None,
    "prefill_4096q_64k": 256,
    "decode_b2_1m_fp8kv_clustered": None,
}

_WL = {}


def workload(sp):
    if sp.name not in _WL:
        _WL[sp.name] = W.make_workload(sp)
    return _WL[sp.name]


def out_dtype(sp):
    return "f32" if sp.kv_dtype == "f32" else "bf16"


def run_fused(wl, dev="cuda"):
    sp = wl.spec
    cache, queries = api.upload(wl, dev)
    idx = torch.full((wl.n_q, sp.top_k), -7, dtype=torch.int32, device=dev)
    ws = api.workspace(api.workspace_size(cache, queries, sp.top_k, _abi.SA_WS_DECODE), dev)
    out, lse, _ = api.decode(cache, queries, sp.top_k, idx=idx, out_dtype=out_dtype(sp), ws=ws)
    st = api.device_status(ws)
    return {"idx": idx.cpu().numpy(), "out": out.float().cpu().numpy(),
            "lse": lse.cpu().numpy(), "status": st}


def sample_rows(wl):
    n = SAMPLES.get(wl.spec.name)
    return np.arange(wl.n_q) if n is None else W.stratified_rows(wl.n_q, n)


@pytest.mark.parametrize("sp", W.CONFIGS, ids=[s.name for s in W.CONFIGS])
def test_decode_matches_oracle(sp):
    wl = workload(sp)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    rows = sample_rows(wl)
    sub = W.subset_queries(wl, rows)
    scores = oracle.index_scores(sub)
    topk = parity.check_topk(res["idx"][rows], scores, sub.visible, sp.top_k)
    ref_out, ref_lse = oracle.sparse_attn(sub, res["idx"][rows])
    err = parity.check_attention(res["out"][rows], ref_out, sp.kv_dtype)
    lse_err = parity.check_lse(res["lse"][rows], ref_lse)
    print(f"\n{sp.name}: rows={len(rows)} swaps={topk['swaps']} "
          f"window={topk['worst_window_fraction']:.3g} max_abs={err['max_abs']:.3g} "
          f"mean_rel={err['mean_rel']:.3g} lse={lse_err:.3g}")
    assert np.all(np.isfinite(res["out"])) and np.all(np.isfinite(res["lse"]))


@pytest.mark.parametrize("sp", W.CONFIGS[:2], ids=[s.name for s in W.CONFIGS[:2]])
def test_unfused_chain_equals_fused_and_topk_is_exact(sp):
    wl = workload(sp)
    fused = run_fused(wl)
    cache, queries = api.upload(wl)
    scores = api.indexer_score(cache, queries)
    valid = torch.from_numpy(wl.visible).cuda()
    idx = api.topk(scores, valid, sp.top_k, wl.max_visible)
    out, lse = api.sparse_mla_attn(cache, queries, idx, sp.top_k, out_dtype=out_dtype(sp))
    s = scores.cpu().numpy().astype(np.float64)
    # scores against the oracle
    ref = oracle.index_scores(wl)
    for t in range(wl.n_q):
        V = wl.visible[t]
        rel = np.abs(s[t, :V] - ref[t, :V]).max() / np.abs(ref[t, :V]).max()
        assert rel <= 1e-4, (t, rel)
    # the top-K kernel is exact on its own fp32 input
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(s, wl.visible, sp.top_k))
    # unfused chain == fused path, bit for bit
    assert np.array_equal(idx.cpu().numpy(), fused["idx"])
    assert np.array_equal(out.float().cpu().numpy(), fused["out"])
    assert np.array_equal(lse.cpu().numpy(), fused["lse"])


def test_topk_exact_on_ties_signed_zeros_and_short_rows():
    rng = np.random.default_rng(7)
    n_q, L, K = 9, 70000, 2048
    s = np.round(rng.standard_normal((n_q, L)), 2).astype(np.float32)
    s[1] = 0.0                                  # all equal: lowest positions win
    s[2, ::2] = -0.0                            # signed zeros tie with +0
    s[2, 1::2] = 0.0
    s[3] = -np.abs(s[3])                        # all negative
    s[4, :] = 1.0
    s[4, 5000:5000 + K] = 2.0                   # a block that is exactly the top-K
    valid = np.array([L, L, L, L, L, 1, K - 1, K, K + 1], np.int32)
    scores = torch.from_numpy(s).cuda()
    idx = api.topk(scores, torch.from_numpy(valid).cuda(), K, L).cpu().numpy()
    ref = oracle.topk(s.astype(np.float64), valid, K)
    assert np.array_equal(idx, ref)
    assert np.array_equal(idx[1], np.arange(K))
    assert np.array_equal(idx[4], np.arange(5000, 5000 + K))


def test_ragged_contexts_around_k_and_page_edges():
    sp = W.WorkloadSpec(name="ragged", seed=21, batch=8,
                        seq_len=("list", (1, 63, 64, 65, 2047, 2048, 2049, 9000)))
    wl = workload(sp)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    parity.check_topk(res["idx"], scores, wl.visible, sp.top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    parity.check_attention(res["out"], ref_out, sp.kv_dtype)
    parity.check_lse(res["lse"], ref_lse)
    assert np.all(res["idx"][0, 1:] == -1) and res["idx"][0, 0] == 0


def test_deterministic_and_independent_of_page_placement():
    wl = workload(W.DECODE_B8_8K)
    a = run_fused(wl)
    b = run_fused(wl)
    c = run_fused(W.permute_pages(wl, seed=5))
    for k in ("idx", "out", "lse"):
        assert np.array_equal(a[k], b[k]), k
        assert np.array_equal(a[k], c[k]), k


@pytest.mark.parametrize("tile,heads", [((0, 0), 128), ((1, 128), 128), ((1, 128), 64),
                                        ((16, 256), 128)])
def test_fp8_latent_cache_small(tile, heads):
    """e4m3 latent with one scale per page or per finer tile (the pages'
    per-token, per-128-element blocks are (1, 128)); 128 heads take the
    tensor-core attention, 64 the CUDA-core one."""
    sp = W.WorkloadSpec(name=f"fp8kv_small_{tile[0]}_{tile[1]}_{heads}", seed=22, batch=3,
                        seq_len=("list", (700, 3000, 5000)), kv_dtype="e4m3",
                        keys=("clusters", 2, 256), kv_scale_tile=tile, heads=heads)
    wl = workload(sp)
    res = run_fused(wl)
    scores = oracle.index_scores(wl)
    parity.check_topk(res["idx"], scores, wl.visible, sp.top_k)
    ref_out, _ = oracle.sparse_attn(wl, res["idx"])
    parity.check_attention(res["out"], ref_out, "e4m3")


@pytest.mark.parametrize("h_index,d_index", [(64, 128), (8, 32)])
def test_bf16_indexer_path(h_index, d_index):
    """The indexer's BF16 path (unscaled bf16 query and keys): the tensor-core
    kernel for 64 heads x 128 dims, the CUDA-core one for other shapes.  bf16
    products are exact in fp32, so the unfused scores must match the oracle's
    to fp32 accumulation error."""
    sp = W.WorkloadSpec(name=f"bf16_index_{h_index}_{d_index}", seed=41, batch=3,
                        seq_len=("list", (900, 2048, 5000)), index_dtype="bf16",
                        h_index=h_index, d_index=d_index, keys=("planted", 0.05, 3.0))
    wl = workload(sp)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    topk = parity.check_topk(res["idx"], scores, wl.visible, sp.top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    err = parity.check_attention(res["out"], ref_out, "bf16")
    parity.check_lse(res["lse"], ref_lse)
    cache, queries = api.upload(wl)
    got = api.indexer_score(cache, queries).cpu().numpy()
    ok = ~np.isnan(scores)
    rel = float(np.abs(got[ok] - scores[ok]).max() / np.abs(scores[ok]).max())
    print(f"\nbf16 index {h_index}x{d_index}: score err {rel:.3g} of max|I|, "
          f"swaps={topk['swaps']} max_abs={err['max_abs']:.3g}")
    assert rel <= 1e-4


@pytest.mark.parametrize("h_index,d_index", [(64, 128), (8, 64)])
def test_mxfp8_indexer_path(h_index, d_index):
    """The pages' MXFP8 index path (e4m3 query and keys, one E8M0 scale per 32
    values): block-scaled tensor-core MMAs for 64 heads x 128 dims, the
    CUDA-core kernel for other shapes.  Products of e4m3 values and powers of
    two are exact in fp32, so the unfused scores must match the oracle's to
    fp32 accumulation error; the fused decode must pass the top-K window and
    the attention tolerances."""
    sp = W.WorkloadSpec(name=f"mxfp8_index_{h_index}_{d_index}", seed=43, batch=4,
                        seq_len=("list", (130, 900, 2049, 5000)), index_dtype="mxfp8",
                        h_index=h_index, d_index=d_index, keys=("planted", 0.05, 3.0))
    wl = workload(sp)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    topk = parity.check_topk(res["idx"], scores, wl.visible, sp.top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    err = parity.check_attention(res["out"], ref_out, "bf16")
    parity.check_lse(res["lse"], ref_lse)
    cache, queries = api.upload(wl)
    got = api.indexer_score(cache, queries).cpu().numpy()
    ok = ~np.isnan(scores)
    rel = float(np.abs(got[ok] - scores[ok]).max() / np.abs(scores[ok]).max())
    print(f"\nmxfp8 index {h_index}x{d_index}: score err {rel:.3g} of max|I|, "
          f"swaps={topk['swaps']} max_abs={err['max_abs']:.3g}")
    assert rel <= 1e-4


def test_mxfp8_headline_decode_matches_oracle():
    """The headline decode (64 sequences, 16K-32K context, planted keys) with the
    MXFP8 index path, every query checked: the launch bench.py times for it."""
    wl = workload(W.DECODE_B64_MXFP8_INDEX)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    topk = parity.check_topk(res["idx"], scores, wl.visible, wl.spec.top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    err = parity.check_attention(res["out"], ref_out, "bf16")
    parity.check_lse(res["lse"], ref_lse)
    print(f"\nmxfp8 headline: swaps={topk['swaps']} window={topk['worst_window_fraction']:.3g} "
          f"max_abs={err['max_abs']:.3g} mean_rel={err['mean_rel']:.3g}")


def test_prefill_query_groups_match_single_queries():
    """Chunked prefill with the query-group promise (q_group = 4: four
    consecutive queries share every key tile, N = 256 MMAs) must give the same
    scores, selection and output as one query at a time, bit for bit, including
    a last group of two queries."""
    sp = W.WorkloadSpec(name="prefill_groups", seed=45, batch=1, seq_len=("fixed", 6000),
                        queries=("prefill", 2900, 38), keys=("planted", 0.05, 3.0))
    wl = workload(sp)
    cache, queries = api.upload(wl)
    assert queries.q_group == 4
    single = dataclasses.replace(queries, q_group=1)
    s4 = api.indexer_score(cache, queries).cpu().numpy()
    s1 = api.indexer_score(cache, single).cpu().numpy()
    for t in range(wl.n_q):
        V = int(wl.visible[t])
        assert np.array_equal(s4[t, :V], s1[t, :V]), t
    outs = []
    for q in (queries, single):
        idx = torch.empty((wl.n_q, sp.top_k), dtype=torch.int32, device="cuda")
        ws = api.workspace(api.workspace_size(cache, q, sp.top_k, _abi.SA_WS_DECODE))
        out, lse, _ = api.decode(cache, q, sp.top_k, idx=idx, ws=ws)
        assert api.device_status(ws) == (_abi.SA_OK, 0)
        outs.append((idx.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()))
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)
    scores = oracle.index_scores(wl)
    parity.check_topk(outs[0][0], scores, wl.visible, sp.top_k)


def test_query_group_mixing_sequences_is_reported():
    """A q_group = 4 promise that the queries break (four different sequences
    in one group) is reported on the device, not scored against the wrong keys."""
    wl = workload(W.DECODE_B8_8K)
    cache, queries = api.upload(wl)
    bad = dataclasses.replace(queries, q_group=4)
    ws = api.workspace(api.workspace_size(cache, bad, wl.spec.top_k, _abi.SA_WS_DECODE))
    api.decode(cache, bad, wl.spec.top_k, ws=ws)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_POSITION)


# ------------------------------------------------------- long contexts ---
# Rows longer than 64K positions take the multi-CTA top-K (count, threshold,
# emit): a batch mixing a row shorter than K, which falls back to the row-wise
# select, with two long rows; massive ties in a long row; and an unmapped page
# inside a long row.
LONG = W.WorkloadSpec(name="long_rows_mixed", seed=47, batch=3,
                      seq_len=("list", (1500, 70000, 140000)), keys=("planted", 0.05, 3.0))


def test_long_rows_match_oracle():
    wl = workload(LONG)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    parity.check_topk(res["idx"], scores, wl.visible, LONG.top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    parity.check_attention(res["out"], ref_out, LONG.kv_dtype)
    parity.check_lse(res["lse"], ref_lse)
    # the unfused top-K on the fused path's own scores picks the same set
    cache, queries = api.upload(wl)
    s = api.indexer_score(cache, queries)
    idx = api.topk(s, torch.from_numpy(wl.visible).cuda(), LONG.top_k, wl.max_visible)
    assert np.array_equal(idx.cpu().numpy(), res["idx"])


@pytest.mark.parametrize("top_k", [1000, 16])
def test_long_rows_other_k(top_k):
    """K = 1000 (rows padded to whole 64-row tiles for the attention) and K = 16
    (more 8K-position chunks than K slots: the row-wise select takes the row)."""
    sp = dataclasses.replace(LONG, name=f"long_rows_k{top_k}", top_k=top_k)
    wl = workload(sp)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    parity.check_topk(res["idx"], scores, wl.visible, top_k)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    parity.check_attention(res["out"], ref_out, sp.kv_dtype)
    parity.check_lse(res["lse"], ref_lse)


def test_long_rows_with_massive_ties_take_lowest_positions():
    wl = workload(LONG)
    k = wl.k_index.copy()
    valid = np.isfinite(wl.k_index_scale)
    rng = np.random.default_rng(6)
    protos = rng.integers(0, 0x7E, size=(3, LONG.d_index), dtype=np.uint8)
    k[valid] = protos[rng.integers(0, 3, size=valid.sum())]
    scale = np.where(valid, np.float32(0.01), wl.k_index_scale).astype(np.float32)
    wl = dataclasses.replace(wl, k_index=k, k_index_scale=scale)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    ref = oracle.topk(oracle.index_scores(wl), wl.visible, LONG.top_k)
    assert np.array_equal(res["idx"], ref)


def test_long_row_unmapped_page_is_reported_and_skipped():
    """An unmapped page inside a long row: reported, none of its positions
    selected, and the attention over the rest matches the oracle."""
    wl = workload(LONG)
    base = run_fused(wl)
    t = 2
    page = int(base["idx"][t, 0]) // 64          # a page holding a selected position
    cache, queries = api.upload(wl)
    cache.page_table[int(wl.q_seq[t]), page] = wl.num_pages + 5
    idx = torch.full((wl.n_q, LONG.top_k), -7, dtype=torch.int32, device="cuda")
    ws = api.workspace(api.workspace_size(cache, queries, LONG.top_k, _abi.SA_WS_DECODE))
    out, lse, _ = api.decode(cache, queries, LONG.top_k, idx=idx, ws=ws)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_PAGE)
    got = idx.cpu().numpy()
    assert not np.any(got[t] // 64 == page) and np.all(got[t] >= 0)
    ref_out, ref_lse = oracle.sparse_attn(W.subset_queries(wl, np.array([t])), got[t:t + 1])
    parity.check_attention(out.float().cpu().numpy()[t:t + 1], ref_out, LONG.kv_dtype)
    parity.check_lse(lse.cpu().numpy()[t:t + 1], ref_lse)


# ------------------------------------------------ device-side data errors ---

def test_bad_page_id_is_reported_not_faulted():
    wl = workload(W.DECODE_B8_8K)
    cache, queries = api.upload(wl)
    cache.page_table[3, 5] = wl.num_pages + 3
    out, lse, _ = api.decode(cache, queries, wl.spec.top_k)
    ws = api.workspace(api.workspace_size(cache, queries, wl.spec.top_k, _abi.SA_WS_DECODE))
    api.decode(cache, queries, wl.spec.top_k, ws=ws)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_PAGE)
    # a clean call on the same workspace clears the word
    cache.page_table[3, 5] = int(wl.page_table[3, 5])
    api.decode(cache, queries, wl.spec.top_k, ws=ws)
    assert api.device_status(ws) == (_abi.SA_OK, 0)


def test_bad_query_position_is_reported():
    wl = workload(W.DECODE_B8_8K)
    cache, queries = api.upload(wl)
    queries.q_pos[2] = int(wl.seq_len[2])           # one past the cached tokens
    ws = api.workspace(api.workspace_size(cache, queries, wl.spec.top_k, _abi.SA_WS_DECODE))
    out, lse, _ = api.decode(cache, queries, wl.spec.top_k, ws=ws)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_POSITION)
    assert torch.isfinite(out.float()).all()


def test_selected_index_outside_visible_range_is_reported():
    wl = workload(W.DECODE_B8_8K)
    cache, queries = api.upload(wl)
    idx = torch.zeros((wl.n_q, 16), dtype=torch.int32, device="cuda")
    idx[1, 3] = int(wl.q_pos[1]) + 1
    ws = api.workspace(api.workspace_size(cache, queries, 16, _abi.SA_WS_ATTN))
    api.sparse_mla_attn(cache, queries, idx, 16, ws=ws)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_INDEX)


def test_empty_batch_is_a_no_op():
    wl = workload(W.TINY)
    cache, queries = api.upload(wl)
    empty = dataclasses.replace(queries, q_seq=queries.q_seq[:0], q_pos=queries.q_pos[:0],
                                q_index=queries.q_index[:0], w=queries.w[:0], q=queries.q[:0])
    out, lse, _ = api.decode(cache, empty, wl.spec.top_k, out_dtype="f32")
    torch.cuda.synchronize()
    assert out.shape[0] == 0


def test_attention_on_unsorted_indices_with_holes():
    """sa_sparse_mla_attn takes any index order and skips -1 entries."""
    wl = workload(W.DECODE_B8_8K)
    K = 700
    rng = np.random.default_rng(31)
    idx = np.full((wl.n_q, K), -1, np.int32)
    for t in range(wl.n_q):
        n = [700, 650, 33, 1, 64, 699, 320, 17][t]
        pos = rng.choice(int(wl.visible[t]), size=n, replace=False).astype(np.int32)
        slots = np.sort(rng.choice(K, size=n, replace=False))
        idx[t, slots] = pos                     # unsorted positions, -1 holes anywhere
    cache, queries = api.upload(wl)
    out, lse = api.sparse_mla_attn(cache, queries, torch.from_numpy(idx).cuda(), K)
    ref_out, ref_lse = oracle.sparse_attn(wl, idx)
    parity.check_attention(out.float().cpu().numpy(), ref_out, "bf16")
    parity.check_lse(lse.cpu().numpy(), ref_lse)


def test_attention_with_large_logits_rescales_output():
    """Queries scaled by 16 (exact in bf16): each head's running maximum jumps
    by far more than 2^8 between key tiles, so the kernel must rescale the
    partial output it keeps on the tensor cores' accumulator."""
    wl = workload(W.DECODE_B8_8K)
    qf = (wl.q.astype(np.uint32) << 16).view(np.float32) * np.float32(16.0)
    wl = dataclasses.replace(wl, q=W.to_bf16_bits(qf))
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    ref_out, ref_lse = oracle.sparse_attn(wl, res["idx"])
    parity.check_attention(res["out"], ref_out, "bf16")
    parity.check_lse(res["lse"], ref_lse)


@pytest.mark.parametrize("pattern", ["all_zero", "three_values"])
def test_fused_topk_on_massive_ties(pattern):
    """All-equal or few-valued scores: the fused top-K must still pick the
    lowest positions among ties (exercising its exact tie-bucket select and
    its fall-back to the row-wise select when the tie bucket overflows)."""
    sp = W.WorkloadSpec(name=f"ties_{pattern}", seed=23, batch=4,
                        seq_len=("list", (3000, 7000, 9000, 30000)))
    wl = W.make_workload(sp)
    k = wl.k_index.copy()
    valid = np.isfinite(wl.k_index_scale)                  # written (non-poisoned) slots
    if pattern == "all_zero":
        k[valid] = 0                                       # e4m3 code 0: every score is 0
    else:
        rng = np.random.default_rng(5)
        protos = rng.integers(0, 0x7E, size=(3, sp.d_index), dtype=np.uint8)
        pick = rng.integers(0, 3, size=valid.sum())
        k[valid] = protos[pick]
    scale = np.where(valid, np.float32(0.01), wl.k_index_scale).astype(np.float32)
    wl = dataclasses.replace(wl, k_index=k, k_index_scale=scale)
    res = run_fused(wl)
    assert res["status"] == (_abi.SA_OK, 0)
    scores = oracle.index_scores(wl)
    ref = oracle.topk(scores, wl.visible, sp.top_k)
    # with exact ties the only correct answer is the oracle's (lower positions win)
    assert np.array_equal(res["idx"], ref)
