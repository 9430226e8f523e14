"""Context-parallel decode kernels on one GPU: G ranks' shards driven in
lockstep from one process (the all-gathers are stacks of the ranks' tensors;
no kernel waits on another rank's), against the single-GPU fused decode.

The merged selection must equal sa_decode's bit for bit (a position's score
does not depend on its shard); the combined output must pass the oracle's
check on that selection and stay within bf16 rounding of sa_decode's output.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from indexed_sparse_attention_lightning_b200 import _abi, api, cp
from indexed_sparse_attention_lightning_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def run_cp(wl, world):
    ops = cp.GpuOps()
    K = wl.spec.top_k
    states = []
    for sh in cp.partition(wl.seq_len, world):
        loc = W.shard_workload(wl, sh.lo, sh.hi)
        cache, queries = api.upload(loc)
        states.append(cp.RankState(cache, queries,
                                   torch.from_numpy(sh.lo[wl.q_seq]).cuda(),
                                   torch.from_numpy(sh.hi[wl.q_seq]).cuda()))
    cands = [cp.phase_candidates(ops, st, K) for st in states]
    score_all = torch.stack([c[0] for c in cands])
    pos_all = torch.stack([c[1] for c in cands])
    parts = [cp.phase_attend(ops, st, score_all, pos_all, K) for st in states]
    for p in parts[1:]:
        assert torch.equal(p[0], parts[0][0])          # every rank merged the same selection
    o_all = torch.stack([p[1] for p in parts])
    lse_all = torch.stack([p[2] for p in parts])
    out, lse = cp.phase_combine(ops, o_all, lse_all, "bf16")
    torch.cuda.synchronize()
    return parts[0][0].cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(), cands


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_context_parallel_decode_matches_single_gpu(world, kv_dtype):
    sp = W.WorkloadSpec(name=f"cp_{kv_dtype}", seed=29, batch=4,
                        seq_len=("list", (5000, 9000, 20000, 33000)), kv_dtype=kv_dtype,
                        keys=("clusters", 4, 512), kv_scale_tile=(1, 128) if kv_dtype == "e4m3"
                        else (0, 0))
    wl = W.make_workload(sp)
    cache, queries = api.upload(wl)
    ref_idx = torch.empty((wl.n_q, sp.top_k), dtype=torch.int32, device="cuda")
    ws = api.workspace(api.workspace_size(cache, queries, sp.top_k, _abi.SA_WS_DECODE))
    ref_out, ref_lse, _ = api.decode(cache, queries, sp.top_k, idx=ref_idx, ws=ws)
    assert api.device_status(ws) == (_abi.SA_OK, 0)
    idx, out, lse, cands = run_cp(wl, world)
    assert np.array_equal(idx, ref_idx.cpu().numpy())
    ref = ref_out.float().cpu().numpy()
    assert np.abs(out - ref).max() <= 2e-2
    ora_out, ora_lse = oracle.sparse_attn(wl, idx)
    parity.check_attention(out, ora_out, kv_dtype)
    parity.check_lse(lse, ora_lse)
    # each rank's candidates are its own positions, ascending, then padding
    sh = cp.partition(wl.seq_len, world)
    for r, (score, pos) in enumerate(cands):
        p = pos.cpu().numpy()
        for t in range(wl.n_q):
            v = p[t][p[t] >= 0]
            b = wl.q_seq[t]
            assert np.all(np.diff(v) > 0) and np.all((v >= sh[r].lo[b]) & (v < sh[r].hi[b]))


def test_merge_prefers_lower_positions_on_ties_and_pads():
    """Equal scores across ranks: the merge keeps the lowest positions; with
    fewer valid candidates than K it pads with -1."""
    K, n_q = 8, 2
    score = torch.zeros((2, n_q, K), device="cuda")
    pos = torch.tensor([[[0, 1, 2, 3, 4, 5, 6, 7], [0, 2, 4, -1, -1, -1, -1, -1]],
                        [[64, 65, 66, 67, 68, 69, 70, 71], [64, 66, -1, -1, -1, -1, -1, -1]]],
                       dtype=torch.int32, device="cuda")
    score[1, 0, 0] = 1.0                                     # one clear winner on rank 1
    lo = torch.tensor([64, 64], dtype=torch.int32, device="cuda")
    hi = torch.tensor([128, 128], dtype=torch.int32, device="cuda")
    g, l = api.merge_candidates(score, pos, K, lo, hi)
    g, l = g.cpu().numpy(), l.cpu().numpy()
    assert list(g[0]) == [0, 1, 2, 3, 4, 5, 6, 64]
    assert list(l[0]) == [-1] * 7 + [0]
    assert list(g[1]) == [0, 2, 4, 64, 66, -1, -1, -1]
    assert list(l[1]) == [-1, -1, -1, 0, 2, -1, -1, -1]


def test_combine_weights_parts_by_lse_and_skips_empty_parts():
    n_q, H, D = 2, 3, 40
    rng = np.random.default_rng(4)
    o = rng.standard_normal((3, n_q, H, D)).astype(np.float32)
    l = rng.standard_normal((3, n_q, H)).astype(np.float32)
    l[2, 1, :] = -np.inf                                    # a rank with no selected row
    out, lse = api.combine_partials(torch.from_numpy(o).cuda(), torch.from_numpy(l).cuda(),
                                    out_dtype="f32")
    m = l.max(axis=0)
    w = np.exp(l - m)
    ref = (w[..., None] * o).sum(0) / w.sum(0)[..., None]
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(lse.cpu().numpy(), m + np.log(w.sum(0)), rtol=1e-6, atol=1e-6)
