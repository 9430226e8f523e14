"""The N > 1 path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Decode shards as independent replicas (no data-path collective): each rank
draws its own batch, and the job reports the slowest rank's time and every
rank's queries.  The reference arm runs on rank 0 alone."""
import dataclasses
import datetime
import os
import socket
from types import SimpleNamespace

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from indexed_sparse_attention_lightning_b200 import workloads as W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = 1.0 + rank      # rank 1 is the slower one
        e2e_ms = 5.0 - rank       # rank 0 is the slower one end to end
        n_q = 64 + 3 * rank
        results[rank] = bench.reduce_over_ranks(dist, torch.device("cpu"), step_ms, e2e_ms, n_q)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_total_queries():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                           join=True, start_method="spawn")
        got = dict(results)
    for rank in range(world):
        assert got[rank] == (2.0, 5.0, 64.0 + 67.0)


def test_ranks_draw_different_batches_of_the_same_shape():
    sp = W.spec("decode_b8_8k")
    a, b = bench.rank_spec(sp, 0), bench.rank_spec(sp, 1)
    assert a == sp and b.seed != a.seed
    assert dataclasses.replace(b, seed=a.seed) == a


def test_single_rank_reduction_is_the_identity():
    assert bench.reduce_over_ranks(None, torch.device("cpu"), 1.5, 2.5, 7) == (1.5, 2.5, 7.0)


def test_reference_arm_runs_on_rank_zero_only():
    # A non-zero rank returns at once, before it builds a workload or runs the oracle.
    args = SimpleNamespace(workload="tiny_decode_b1_1k_fp32", steps=1, warmup=0)
    assert bench.run_reference(args, rank=1, world=2) == 0
