"""GPU parity for input preparation: the CUDA kernels (through the C ABI)
against the oracle's encoders and scatter.

* query quantisation: codes and scales bit-exact, bf16 and fp32 inputs, the
  vectorised row lengths (128, 256) and the generic ones, up to the prefill
  size (4096 tokens x 64 heads);
* append: every pool bit-exact after the step's tokens are written, for each
  pool format, with invalid tokens skipped and reported;
* a decode step that appends its token and quantises its query on the GPU
  selects and attends like the oracle run on the same prepared inputs.
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


def _inputs(rng, shape, dtype, spread=True):
    """Random values, rows scaled over 2^-6..2^6 when `spread` (else N(0,1), the
    workloads' distribution), the first row all zero; (torch tensor on the GPU,
    the exact fp32 values the kernel sees)."""
    x = rng.standard_normal(shape)
    if spread:
        x = x * np.exp2(rng.uniform(-6, 6, shape[:-1] + (1,)))
    x = x.astype(np.float32)
    x.reshape(-1, shape[-1])[0] = 0.0
    t = torch.from_numpy(x)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
        exact = t.float().numpy()
    else:
        exact = x
    return t.cuda(), exact


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n_q,h,d", [(37, 64, 128), (5, 64, 256), (9, 16, 96), (3, 7, 48),
                                     (4096, 64, 128)])
def test_quantize_index_query_bit_exact(dtype, n_q, h, d):
    rng = np.random.default_rng(n_q * 1000 + d)
    q, exact = _inputs(rng, (n_q, h, d), dtype)
    codes, scales = api.quantize_index_query(q)
    want_codes, want_scales = oracle.quantize_index_query(exact)
    assert np.array_equal(scales.cpu().numpy(), want_scales)
    assert np.array_equal(codes.cpu().numpy(), want_codes)


def test_quantize_index_query_near_rounding_boundaries():
    """Quotients x / scale within a few fp32 units of an e4m3 rounding midpoint,
    with scales whose reciprocal is inexact: the codes must still be those of
    the correctly rounded quotient."""
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    v = np.unique(e4[np.isfinite(e4) & (e4 > 0)]).astype(np.float64)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)                # exact in fp32
    rows = []
    for amax in (447.0, 300.7, 0.0123, 5e-3, 1000.5, 3.3e-7):
        scale = np.float32(amax) / np.float32(448.0)
        vals = (mids * scale).astype(np.float32)                  # x / scale ~ midpoint
        near = [np.nextafter(vals, np.float32(np.inf) if k > 0 else np.float32(-np.inf))
                for k in (1, -1)]
        allv = np.concatenate([vals, near[0], near[1], (v.astype(np.float32) * scale)])
        allv = allv[np.abs(allv) < np.float32(amax)]
        for c0 in range(0, allv.size, 127):
            chunk = allv[c0:c0 + 127]
            row = np.zeros(128, dtype=np.float32)
            row[0] = amax
            row[1:1 + chunk.size] = chunk
            rows.append(row)
    x = np.stack(rows).astype(np.float32)
    x[1::2] *= -1.0
    n = x.shape[0]
    x = np.concatenate([x, np.zeros(((-n) % 64, 128), np.float32)]).reshape(-1, 64, 128)
    codes, scales = api.quantize_index_query(torch.from_numpy(x).cuda())
    want_codes, want_scales = oracle.quantize_index_query(x)
    assert np.array_equal(scales.cpu().numpy(), want_scales)
    assert np.array_equal(codes.cpu().numpy(), want_codes)


def test_quantize_index_query_empty_is_a_no_op():
    q = torch.empty((0, 64, 128), dtype=torch.bfloat16, device="cuda")
    codes, scales = api.quantize_index_query(q)
    assert codes.shape == (0, 64, 128) and scales.shape == (0, 64)


def _bits(a: np.ndarray) -> np.ndarray:
    """Compare pools by bit pattern (f32 pools may hold NaN poison)."""
    return a.view(np.uint32) if a.dtype == np.float32 else a


def _cache_arrays(cache):
    out = {}
    for k in ("k_index", "k_index_scale", "kv", "kv_rope", "kv_scale"):
        t = getattr(cache, k)
        if t is None:
            out[k] = None
            continue
        a = t.cpu().numpy()
        out[k] = a.view(np.uint16) if a.dtype == np.int16 else a
    return out


def _layout(wl):
    sp = wl.spec
    return {"page_table": wl.page_table, "page_size": sp.page_size, "num_pages": wl.num_pages,
            "index_dtype": sp.index_dtype, "kv_dtype": sp.kv_dtype, "d_latent": sp.d_latent,
            "kv_scale_dims": sp.kv_tile[1]}


def _tokens(wl, rng, bad: bool):
    """One token per sequence at its last position, a few more at distinct
    valid positions, and (with `bad`) tokens that must be skipped."""
    seq, pos = [], []
    for b, L in enumerate(wl.seq_len.tolist()):
        seq.append(b)
        pos.append(L - 1)
        for p in rng.choice(L - 1, size=3, replace=False).tolist():
            seq.append(b)
            pos.append(p)
    if bad:
        seq += [-1, wl.seq_len.shape[0], 0, 0]
        pos += [0, 0, -3, wl.max_pages * wl.spec.page_size]
    return np.array(seq, dtype=np.int32), np.array(pos, dtype=np.int32)


SPECS = [
    ("bf16", "e4m3", (0, 0)),
    ("bf16", "bf16", (0, 0)),
    ("f32", "f32", (0, 0)),
    ("e4m3", "e4m3", (1, 128)),
    ("e4m3", "e4m3", (1, 16)),
]


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("kv_dtype,index_dtype,tile", SPECS,
                         ids=[f"{a}-{b}-{c[0]}x{c[1]}" for a, b, c in SPECS])
def test_append_tokens_bit_exact(in_dtype, kv_dtype, index_dtype, tile):
    sp = W.WorkloadSpec(name=f"append_{kv_dtype}_{index_dtype}_{tile[1]}", seed=31, batch=3,
                        seq_len=("list", (200, 1000, 4097)), kv_dtype=kv_dtype,
                        index_dtype=index_dtype, kv_scale_tile=tile, h_index=8, heads=16)
    if kv_dtype == "f32":
        sp = dataclasses.replace(sp, q_dtype="f32")
    wl = W.make_workload(sp)
    cache, _ = api.upload(wl)
    rng = np.random.default_rng(32)
    seq, pos = _tokens(wl, rng, bad=True)
    k_t, k_exact = _inputs(rng, (seq.size, sp.d_index), in_dtype)
    kv_t, kv_exact = _inputs(rng, (seq.size, sp.d_latent + sp.d_rope), in_dtype)
    ws = api.append_tokens(cache, torch.from_numpy(seq).cuda(), torch.from_numpy(pos).cuda(),
                           k_index=k_t, kv=kv_t)
    st, detail = api.device_status(ws)
    assert st == _abi.SA_ERR_DEVICE_FAULT
    assert detail in (_abi.SA_DETAIL_BAD_POSITION, _abi.SA_DETAIL_BAD_PAGE)
    before = {k: getattr(wl, k) for k in ("k_index", "k_index_scale", "kv", "kv_rope",
                                           "kv_scale")}
    want, skipped = oracle.append_tokens(before, _layout(wl), seq, pos, k_exact, kv_exact)
    assert len(skipped) == 4
    got = _cache_arrays(cache)
    for k, a in want.items():
        if a is None:
            assert got[k] is None
            continue
        assert np.array_equal(_bits(got[k]), _bits(a)), k


def test_append_reports_a_bad_page_and_writes_the_rest():
    sp = W.WorkloadSpec(name="append_bad_page", seed=33, batch=2, seq_len=("list", (300, 500)),
                        h_index=8, heads=16)
    wl = W.make_workload(sp)
    wl.page_table[1, 2] = wl.num_pages + 5          # position 128..191 of sequence 1
    cache, _ = api.upload(wl)
    seq = np.array([0, 1, 1], dtype=np.int32)
    pos = np.array([299, 150, 499], dtype=np.int32)
    rng = np.random.default_rng(34)
    k_t, k_exact = _inputs(rng, (3, sp.d_index), "bf16")
    kv_t, kv_exact = _inputs(rng, (3, sp.d_latent + sp.d_rope), "bf16")
    ws = api.append_tokens(cache, torch.from_numpy(seq).cuda(), torch.from_numpy(pos).cuda(),
                           k_index=k_t, kv=kv_t)
    assert api.device_status(ws) == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_PAGE)
    before = {k: getattr(wl, k) for k in ("k_index", "k_index_scale", "kv", "kv_rope",
                                           "kv_scale")}
    want, skipped = oracle.append_tokens(before, _layout(wl), seq, pos, k_exact, kv_exact)
    assert skipped == [(1, "page")]
    got = _cache_arrays(cache)
    for k, a in want.items():
        if a is not None:
            assert np.array_equal(_bits(got[k]), _bits(a)), k
    # valid tokens only: status stays clear
    ws = api.append_tokens(cache, torch.from_numpy(seq[[0, 2]]).cuda(),
                           torch.from_numpy(pos[[0, 2]]).cuda(), k_index=k_t[[0, 2]],
                           kv=kv_t[[0, 2]])
    assert api.device_status(ws) == (_abi.SA_OK, 0)


def test_append_of_no_tokens_is_a_no_op():
    sp = W.WorkloadSpec(name="append_none", seed=37, batch=2, seq_len=("list", (100, 200)),
                        h_index=8, heads=16)
    wl = W.make_workload(sp)
    cache, _ = api.upload(wl)
    before = _cache_arrays(cache)
    none = torch.empty(0, dtype=torch.int32, device="cuda")
    ws = api.append_tokens(cache, none, none,
                           k_index=torch.empty((0, sp.d_index), dtype=torch.bfloat16,
                                               device="cuda"))
    assert api.device_status(ws) == (_abi.SA_OK, 0)
    after = _cache_arrays(cache)
    for k, a in before.items():
        if a is not None:
            assert np.array_equal(_bits(after[k]), _bits(a)), k


def test_prepared_decode_step_matches_oracle():
    """Append each sequence's new token at its last position, quantise the
    step's indexer query, then decode: the GPU and the oracle agree on the
    same prepared inputs."""
    sp = W.WorkloadSpec(name="prepared_step", seed=35, batch=4,
                        seq_len=("list", (1500, 2048, 2049, 6000)))
    wl = W.make_workload(sp)
    cache, queries = api.upload(wl)
    rng = np.random.default_rng(36)
    seq = np.arange(sp.batch, dtype=np.int32)
    pos = (wl.seq_len - 1).astype(np.int32)
    # N(0,1) like the cached rows: the attention tolerances assume outputs of
    # that size (a row scaled by 2^6 would leave bf16 rounding of the output
    # alone above 2e-2)
    k_t, k_exact = _inputs(rng, (sp.batch, sp.d_index), "bf16", spread=False)
    kv_t, kv_exact = _inputs(rng, (sp.batch, sp.d_latent + sp.d_rope), "bf16", spread=False)
    qi_t, qi_exact = _inputs(rng, (wl.n_q, sp.h_index, sp.d_index), "bf16", spread=False)
    ws = api.append_tokens(cache, torch.from_numpy(seq).cuda(), torch.from_numpy(pos).cuda(),
                           k_index=k_t, kv=kv_t)
    assert api.device_status(ws) == (_abi.SA_OK, 0)
    api.quantize_index_query(qi_t, out=queries.q_index, scale=queries.q_index_scale)
    idx = torch.full((wl.n_q, sp.top_k), -7, dtype=torch.int32, device="cuda")
    ws = api.workspace(api.workspace_size(cache, queries, sp.top_k, _abi.SA_WS_DECODE))
    out, lse, _ = api.decode(cache, queries, sp.top_k, idx=idx, out_dtype="bf16", ws=ws)
    assert api.device_status(ws) == (_abi.SA_OK, 0)

    before = {k: getattr(wl, k) for k in ("k_index", "k_index_scale", "kv", "kv_rope",
                                           "kv_scale")}
    pools, skipped = oracle.append_tokens(before, _layout(wl), seq, pos, k_exact, kv_exact)
    assert skipped == []
    codes, scales = oracle.quantize_index_query(qi_exact)
    ref = dataclasses.replace(wl, q_index=codes, q_index_scale=scales, **pools)
    scores = oracle.index_scores(ref)
    # the appended token is visible to its own query
    assert np.all(np.isfinite(scores[np.arange(wl.n_q), wl.q_pos]))
    gpu_idx = idx.cpu().numpy()
    parity.check_topk(gpu_idx, scores, ref.visible, sp.top_k)
    ref_out, ref_lse = oracle.sparse_attn(ref, gpu_idx)
    parity.check_attention(out.float().cpu().numpy(), ref_out, "bf16")
    parity.check_lse(lse.cpu().numpy(), ref_lse)
