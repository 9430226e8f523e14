"""Context-parallel decode on CPU: the partition, the shard caches, and a step
over two gloo ranks on 127.0.0.1 against the single-rank result.

The ranks run the library's orchestration (``cp.decode_step``: two
all-gathers around the compute steps) with the compute steps taken by the
fp64 oracle, so what is checked here is the partition, the shard layout, the
exchange, the candidate merge rule and the lse merge; the GPU kernels of those
steps are checked against the single-GPU decode in ``test_gpu_cp.py``.
"""
import dataclasses
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from indexed_sparse_attention_lightning_b200 import cp
from indexed_sparse_attention_lightning_b200 import workloads as W


def small_spec(**kw):
    base = dict(name="cp_small", seed=13, batch=2, seq_len=("list", (1000, 1411)),
                h_index=4, d_index=16, index_dtype="e4m3", top_k=96, heads=3, d_latent=24,
                d_rope=8, kv_dtype="bf16", q_dtype="bf16", keys=("planted", 0.05, 3.0))
    base.update(kw)
    return W.WorkloadSpec(**base)


def test_partition_is_contiguous_and_page_aligned():
    L = np.array([64 * 7 + 5, 64 * 3, 1 << 20])
    shards = cp.partition(L, 3)
    for b in range(3):
        assert shards[0].lo[b] == 0 and shards[-1].hi[b] == L[b]
        for r in range(3):
            assert shards[r].lo[b] % 64 == 0 and shards[r].hi[b] > shards[r].lo[b]
            if r:
                assert shards[r].lo[b] == shards[r - 1].hi[b]
    with pytest.raises(ValueError):
        cp.partition([64 * 2], 3)  # fewer pages than ranks


@pytest.mark.parametrize("world", [2, 3])
def test_shards_hold_the_same_rows_under_local_positions(world):
    wl = W.make_workload(small_spec())
    for sh in cp.partition(wl.seq_len, world):
        loc = W.shard_workload(wl, sh.lo, sh.hi)
        for b in range(wl.seq_len.shape[0]):
            s = np.arange(sh.hi[b] - sh.lo[b])
            lrow = loc.page_table[b][s // 64].astype(np.int64) * 64 + s % 64
            g = s + sh.lo[b]
            grow = wl.page_table[b][g // 64].astype(np.int64) * 64 + g % 64
            assert np.array_equal(loc.k_index.reshape(-1, 16)[lrow], wl.k_index.reshape(-1, 16)[grow])
            assert np.array_equal(loc.kv.reshape(-1, 32)[lrow], wl.kv.reshape(-1, 32)[grow])
        assert np.array_equal(loc.q_pos, sh.hi[loc.q_seq] - sh.lo[loc.q_seq] - 1)


class OracleOps:
    """The compute steps on the CPU by the fp64 oracle (test stand-in for
    cp.GpuOps); ``cache`` is the rank's shard workload."""

    def candidates(self, wl, _queries, top_k, lo):
        s = oracle.index_scores(wl)
        idx = oracle.topk(s, wl.visible, top_k)
        score = np.where(idx >= 0, np.take_along_axis(s, np.maximum(idx, 0), 1), -np.inf)
        pos = np.where(idx >= 0, idx + lo.numpy()[:, None], -1)
        return torch.from_numpy(score), torch.from_numpy(pos.astype(np.int32))

    def merge(self, score_all, pos_all, top_k, lo, hi):
        sc, ps = score_all.numpy(), pos_all.numpy()
        n_q = sc.shape[1]
        g = np.full((n_q, top_k), -1, np.int32)
        loc = np.full((n_q, top_k), -1, np.int32)
        for t in range(n_q):
            s, p = sc[:, t].ravel(), ps[:, t].ravel()
            ok = p >= 0
            s, p = s[ok], p[ok]
            order = np.lexsort((p, -s))[:top_k]      # score desc, then lower position
            sel = np.sort(p[order])
            g[t, :sel.size] = sel
            inside = (sel >= int(lo[t])) & (sel < int(hi[t]))
            loc[t, :sel.size] = np.where(inside, sel - int(lo[t]), -1)
        return torch.from_numpy(g), torch.from_numpy(loc)

    def attend(self, wl, _queries, idx_local, top_k):
        out, lse = oracle.sparse_attn(wl, idx_local.numpy())
        return torch.from_numpy(out), torch.from_numpy(lse)

    def combine(self, o_all, lse_all, _out_dtype):
        o, l = o_all.numpy(), lse_all.numpy()
        m = np.max(l, axis=0)
        w = np.where(np.isfinite(l), np.exp(l - m), 0.0)
        tot = w.sum(axis=0)
        out = (w[..., None] * o).sum(axis=0) / tot[..., None]
        return torch.from_numpy(out), torch.from_numpy(m + np.log(tot))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.make_workload(small_spec())
        sh = cp.partition(wl.seq_len, world)[rank]
        loc = W.shard_workload(wl, sh.lo, sh.hi)
        st = cp.RankState(loc, None, torch.from_numpy(sh.lo[wl.q_seq]),
                          torch.from_numpy(sh.hi[wl.q_seq]))
        out, lse, idx = cp.decode_step(cp.TorchComm(), OracleOps(), st, wl.spec.top_k)
        results[rank] = (out.numpy(), lse.numpy(), idx.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_single_rank_decode():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        ps = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(timeout=240)
            assert p.exitcode == 0
        res = dict(results)
    wl = W.make_workload(small_spec())
    idx_ref = oracle.topk(oracle.index_scores(wl), wl.visible, wl.spec.top_k)
    out_ref, lse_ref = oracle.sparse_attn(wl, idx_ref)
    for r in range(world):
        out, lse, idx = res[r]
        assert np.array_equal(idx, idx_ref)                  # the same selection everywhere
        np.testing.assert_allclose(out, out_ref, rtol=0, atol=1e-10)
        np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-10)
    # both shards contribute to the selection
    sh = cp.partition(wl.seq_len, world)
    for b in range(wl.seq_len.shape[0]):
        sel = idx_ref[b][idx_ref[b] >= 0]
        assert np.any(sel < sh[0].hi[b]) and np.any(sel >= sh[1].lo[b])
