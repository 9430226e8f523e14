"""Context-parallel decode across GPUs (one process per GPU).

One long sequence is split along its context: rank r of G holds positions
[lo_r, hi_r) of every sequence -- a contiguous, page-aligned share -- in its own
paged caches ("Inference Acceleration for New Large Model Architectures"
§5.1-5.2: each device handles a contiguous portion of the sequence; "Long-
Context LLM Inference Optimization", Distributed Scaling).  A decode step is
two exchanges around the library's kernels:

  1. each rank scores its positions and keeps its own top-K
     (``sa_local_candidates``: K (score, global position) pairs per query);
  2. all-gather of the candidates (K x 8 bytes per query per rank);
  3. every rank merges them into the same global top-K and keeps the part it
     holds (``sa_merge_candidates``);
  4. each rank attends over its part (``sa_sparse_mla_attn``, fp32 partial
     output and log-sum-exp);
  5. all-gather of the partial outputs and lse;
  6. the partials are merged by their lse (``sa_combine_partials``).

The selected positions equal the single-GPU ``sa_decode``'s exactly: a
position's score does not depend on the shard that computes it, and the merge
keeps the same ties (score, then lower position).  The output differs from the
single-GPU one only by the rounding of the lse merge.

The collectives are the caller's: ``comm.all_gather(t)`` returns the ranks'
tensors stacked rank-major ([world, *t.shape]); ``TorchComm`` does it with
``torch.distributed`` (NCCL on GPUs).  The compute steps go through ``ops``;
``GpuOps`` runs them on this GPU through the C ABI.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import api


@dataclass(frozen=True)
class Shard:
    """Positions [lo[b], hi[b]) of sequence b held by rank ``rank`` of ``world``."""

    rank: int
    world: int
    lo: np.ndarray  # int32 [batch]
    hi: np.ndarray  # int32 [batch]


def partition(seq_len, world: int, page_size: int = 64) -> list:
    """Split every sequence's pages as evenly as whole pages allow: rank r of G
    holds pages [P r / G, P (r + 1) / G) of a sequence with P pages.  Every
    rank must hold at least one page of every sequence."""
    L = np.asarray(seq_len, dtype=np.int64)
    P = (L + page_size - 1) // page_size
    if world < 1 or np.any(P < world):
        raise ValueError("every sequence needs at least one page per rank")
    out = []
    for r in range(world):
        lo = np.minimum(P * r // world * page_size, L)
        hi = np.minimum(P * (r + 1) // world * page_size, L)
        out.append(Shard(r, world, lo.astype(np.int32), hi.astype(np.int32)))
    return out


class TorchComm:
    """All-gather over a ``torch.distributed`` process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        flat = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                           device=t.device)
        self.dist.all_gather_into_tensor(flat, t, group=self.group)
        return flat.view((self.world,) + tuple(t.shape))


class GpuOps:
    """The compute steps on this GPU, through the library's C ABI."""

    def candidates(self, cache, queries, top_k: int, lo: torch.Tensor):
        score, pos, _ = api.local_candidates(cache, queries, top_k, lo)
        return score, pos

    def merge(self, score_all, pos_all, top_k: int, lo: torch.Tensor, hi: torch.Tensor):
        return api.merge_candidates(score_all, pos_all, top_k, lo, hi)

    def attend(self, cache, queries, idx_local, top_k: int):
        return api.sparse_mla_attn(cache, queries, idx_local, top_k, out_dtype="f32")

    def combine(self, o_all, lse_all, out_dtype: str):
        return api.combine_partials(o_all, lse_all, out_dtype=out_dtype)


@dataclass
class RankState:
    """One rank's part of a step: its shard's cache and queries (query
    positions local to the shard: its last position for decode) and the
    shard's global range for each query's sequence (int32 [n_q], on the
    rank's device)."""

    cache: object
    queries: object
    lo: torch.Tensor
    hi: torch.Tensor


# The step in three phases between the two exchanges, so that a caller that
# drives several ranks from one thread (tests) can run them in lockstep.
def phase_candidates(ops, st: RankState, top_k: int):
    return ops.candidates(st.cache, st.queries, top_k, st.lo)


def phase_attend(ops, st: RankState, score_all, pos_all, top_k: int):
    idx_global, idx_local = ops.merge(score_all, pos_all, top_k, st.lo, st.hi)
    o, lse = ops.attend(st.cache, st.queries, idx_local, top_k)
    return idx_global, o, lse


def phase_combine(ops, o_all, lse_all, out_dtype: str):
    return ops.combine(o_all, lse_all, out_dtype)


def decode_step(comm, ops, st: RankState, top_k: int, out_dtype: str = "bf16"):
    """One context-parallel decode step on this rank.  Returns (out, lse,
    global top-K positions), the same on every rank."""
    score, pos = phase_candidates(ops, st, top_k)
    score_all, pos_all = comm.all_gather(score), comm.all_gather(pos)
    idx_global, o, lse = phase_attend(ops, st, score_all, pos_all, top_k)
    o_all, lse_all = comm.all_gather(o), comm.all_gather(lse)
    out, lse_out = phase_combine(ops, o_all, lse_all, out_dtype)
    return out, lse_out, idx_global
