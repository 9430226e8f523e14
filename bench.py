#!/usr/bin/env python3
"""Sparse-attention decode throughput on B200: indexer + top-K + sparse MLA attention.

One step = one fused ``sa_decode`` over one batch of synthetic queries (all
three steps of the path).  Prints ONE JSON line (rank 0):

  value     query-tokens/s over all ranks, device time (CUDA events), inputs
            resident in HBM, L2 flushed before every timed step (a 256 MiB
            buffer written, then read back, outside the timed region);
  e2e       the same metric through the public API with host buffers, as a
            serving loop runs a step: pinned host -> device copy of the step's
            inputs (queries in the projection's format and each query's new
            token), quantisation of the indexer query, append of the new tokens,
            the decode, device -> host copy of the outputs, all inside the
            timed region (steps pipelined over three streams, no L2 flush);
  roofline  the dominant phase's algorithmic bytes / its event-timed duration
            against the measured HBM copy bandwidth;
  cpu_baseline  the fp64 oracle on a bounded sample, on this host's cores;
  other_configs the other configurations, each device-timed the same way in
            the same run (step, phases, path bytes, roofline, clocks).

``--impl reference`` times the fp64 oracle instead (rank 0 only).
Multi-GPU (torchrun): every rank decodes its own batch (seeded per rank), no
collective on the data path ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "decode_b64_16k_32k_planted"
METRIC = "sparse-attn decode query-tokens/s (indexer+top-K+SFA); % of HBM roofline"
UNIT = "query-tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (skip the other configurations)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


# --------------------------------------------------------------- helpers ---

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def measured_peaks():
    """(HBM GB/s, dense bf16 TFLOP/s for a kernel timed alone, "measured" or "fallback")."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def algorithmic_flops(wl, idx: np.ndarray) -> dict:
    """Tensor-core work per step, by phase: the indexer does 2 * h_index * d_index
    flops per visible (query, position); the attention 2 * heads * (d_latent + d_rope
    + d_latent) per selected row (Q K^T over 576 dims, P V over 512)."""
    sp = wl.spec
    V = wl.visible.astype(np.int64)
    n_sel = int((idx >= 0).sum())
    return {"indexer": int(V.sum()) * 2 * sp.h_index * sp.d_index,
            "attention": n_sel * 2 * sp.heads * (2 * sp.d_latent + sp.d_rope)}


def roofline(wl, name: str, ms: float, nbytes: dict, flops: dict) -> dict:
    """Roofline of one phase.  Decode (one query per sequence) streams every key
    and selected row once: HBM-bound, algorithmic bytes over the measured copy
    bandwidth.  Chunked prefill (many queries of one sequence) reuses keys and rows
    from L2, so the tensor pipe bounds it: algorithmic flops over the dtype's
    peak (e4m3 = 2 x the measured bf16 GEMM, the nominal fp8:bf16 ratio; the
    indexer's BF16 path and the attention take the bf16 GEMM's)."""
    hbm, bf16, kind = measured_peaks()
    sp = wl.spec
    shared = wl.n_q > wl.seq_len.shape[0]
    secs = ms / 1e3
    if shared and name in flops and sp.index_dtype in ("e4m3", "bf16"):
        fp8 = name == "indexer" and sp.index_dtype == "e4m3"
        peak = bf16 * (2.0 if fp8 else 1.0)
        achieved = flops[name] / secs / 1e12 if secs > 0 else 0.0
        return {"bound": "tensor", "kernel": name, "achieved": achieved, "peak": peak,
                "peak_kind": kind + (" (fp8 = 2 x bf16)" if fp8 else " (bf16)"),
                "unit": "TFLOP/s", "frac": achieved / peak}
    achieved = nbytes[name] / secs / 1e9 if secs > 0 else 0.0
    return {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": hbm,
            "peak_kind": kind, "unit": "GB/s", "frac": achieved / hbm}


def algorithmic_bytes(wl, idx: np.ndarray) -> dict:
    """Bytes the path must move per step, by phase (the metric's definition:
    indexer keys + key scales + selected KV rows + outputs)."""
    sp = wl.spec
    V = wl.visible.astype(np.int64)
    key_b = sp.d_index * {"e4m3": 1, "mxfp8": 1, "bf16": 2, "f32": 4}[sp.index_dtype]
    # one fp32 scale per key, or one E8M0 byte per 32 values (MXFP8)
    scale_b = {"e4m3": 4, "mxfp8": sp.d_index // 32}.get(sp.index_dtype, 0)
    indexer = int((V * (key_b + scale_b)).sum())
    n_sel = np.minimum(V, sp.top_k)
    if sp.kv_dtype == "e4m3":
        # codes + bf16 rope per row, and 4 B per scale tile the selection touches
        row_b = sp.d_latent + 2 * sp.d_rope
        tile_t, tile_d = sp.kv_tile
        tiles = 0
        for t in range(wl.n_q):
            sel = idx[t][idx[t] >= 0]
            tiles += np.unique(sel // tile_t).size * (sp.d_latent // tile_d)
        rows = int((n_sel * row_b).sum()) + 4 * tiles
    else:
        row_b = (sp.d_latent + sp.d_rope) * (2 if sp.kv_dtype == "bf16" else 4)
        rows = int((n_sel * row_b).sum())
    out_b = 2 if sp.kv_dtype != "f32" else 4
    outputs = wl.n_q * sp.heads * (sp.d_latent * out_b + 4)
    return {"indexer": indexer, "topk": 0, "attention": rows + outputs,
            "total": indexer + rows + outputs}


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled DURING the timed
    region by an NVML polling thread (a sample every half millisecond or so;
    it only reads)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []          # (sm_mhz, reason bitmask)
        self.max_mhz = None
        self.thread = None
        self.stop = False

    def _handle(self, nv):
        import torch
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.nv, self.h = nv, h
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            # pay the first-query cost of each call before the timed region
            nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            nv.nvmlDeviceGetCurrentClocksEventReasons(h)

            def poll():
                while not self.stop:
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                        self.samples.append((mhz, rs))
                    except Exception:
                        pass
                    time.sleep(0.0005)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            time.sleep(0.002)
        except Exception:
            self.thread = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return None
        reasons = set()
        for _, rs in self.samples:
            for name, attr in self.REASONS:
                if rs & int(getattr(self.nv, attr, 0)):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml"}


def traffic_for(kernel: str, source_files: list[str], workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    this workload and the kernel's sources are unchanged since; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path)).get(kernel)
    except Exception:
        return None
    if not rec or rec.get("workload") != workload:
        return None
    h = hashlib.sha256()
    for f in source_files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec.get("dram_bytes_per_launch")


# -------------------------------------------------------------- oracle leg ---

def time_oracle(wl, budget_s: float):
    """Run the oracle on a growing sample of queries until ~budget_s is spent."""
    import oracle
    from indexed_sparse_attention_lightning_b200 import workloads as W
    order = W.stratified_rows(wl.n_q, wl.n_q)
    rng = np.random.default_rng(12345)
    order = rng.permutation(order)
    done, spent = 0, 0.0
    while done < len(order) and spent < budget_s:
        sub = W.subset_queries(wl, order[done:done + 1])
        t0 = time.perf_counter()
        oracle.run(sub)
        spent += time.perf_counter() - t0
        done += 1
    return done, spent


def workload_config(sp, wl, world: int) -> dict:
    """The bench line's `config`: the workload by name and its sizes (both arms)."""
    return {
        "workload": sp.name, "batch": int(wl.seq_len.shape[0]), "queries_per_gpu": wl.n_q,
        "context_mean": float(wl.seq_len.mean()), "top_k": sp.top_k, "heads": sp.heads,
        "index_heads": sp.h_index, "index_dim": sp.d_index,
        "index_dtype": sp.index_dtype, "kv_dtype": sp.kv_dtype,
        "page_size": sp.page_size,
        "l2": "flushed before every timed step (256 MiB written, then read back)",
        "parallelism": f"replicas x{world}"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    from indexed_sparse_attention_lightning_b200 import workloads as W
    wl = W.make_workload(W.spec(args.workload))
    import oracle
    cores = oracle.threads()
    rng = np.random.default_rng(777)
    order = rng.permutation(wl.n_q)
    per_step = []
    for k in range(args.warmup + args.steps):
        rows = order[[k % wl.n_q]]
        sub = W.subset_queries(wl, rows)
        t0 = time.perf_counter()
        oracle.run(sub, nthreads=cores)
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            per_step.append(dt)
    total = sum(per_step)
    value = args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": dict(workload_config(wl.spec, wl, world),
                       l2="host memory (the oracle runs on the CPU)",
                       sample="1 query of the workload per step, rotating"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "1 query of the workload per step (fp64 oracle, all steps)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our leg ---

def rank_spec(sp, rank: int):
    """Replicas: every rank decodes its own batch, drawn with its own seed."""
    return sp if rank == 0 else dataclasses.replace(sp, seed=sp.seed + 1000 * rank)


def reduce_over_ranks(dist, device, step_ms: float, e2e_ms: float, n_q: int):
    """(max step time, max end-to-end step time, total queries) over all ranks:
    the job is as slow as its slowest rank and serves every rank's queries."""
    import torch
    t = torch.tensor([step_ms, e2e_ms], dtype=torch.float64, device=device)
    q = torch.tensor([float(n_q)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(q, op=dist.ReduceOp.SUM)
    return float(t[0]), float(t[1]), float(q[0])


def input_prep_bytes(wl, with_kv: bool) -> int:
    """Algorithmic bytes of one step's input preparation: the bf16 indexer query
    read, its e4m3 codes and scales written; per new token the bf16 key read and
    its code row and scale written, and (with_kv) the bf16 latent row read and
    its stored form written."""
    sp = wl.spec
    n, h, d = wl.n_q, sp.h_index, sp.d_index
    b = n * h * d * 2 + n * h * d + n * h * 4
    b += n * (d * 2 + d + 4)
    if with_kv:
        D = sp.d_latent + sp.d_rope
        if sp.kv_dtype == "e4m3":
            stored = sp.d_latent + 2 * sp.d_rope + 4 * (sp.d_latent // sp.kv_tile[1])
        else:
            stored = D * (2 if sp.kv_dtype == "bf16" else 4)
        b += n * (D * 2 + stored)
    return b


def flush_l2(buf):
    """Evict the previous step's data from L2 before a timed step: write a buffer
    larger than L2, then read it back, so that L2 is left holding clean lines and
    the timed step does not pay for writing the flush's own dirty lines back to
    HBM (about 8 us of the indexer's time on the headline workload)."""
    import torch
    buf.zero_()
    buf.view(torch.int64).sum()


def time_input_prep(args, wl, cache, dev, flush):
    """One step's input preparation, timed on its own after the decode timing:
    the indexer query quantised from bf16, and one new token per query (decode's
    newest token, a prefill chunk's tokens) appended at the query's position to
    both caches.  A latent cache with one scale per page cannot take single
    tokens; there only the keys are appended."""
    import torch
    from indexed_sparse_attention_lightning_b200 import api
    sp = wl.spec
    if sp.index_dtype != "e4m3":
        return None
    with_kv = not (sp.kv_dtype == "e4m3" and sp.kv_tile[0] != 1)
    g = torch.Generator(device=dev)
    g.manual_seed(sp.seed + 77)
    qi = torch.randn((wl.n_q, sp.h_index, sp.d_index), generator=g, device=dev).bfloat16()
    k_new = torch.randn((wl.n_q, sp.d_index), generator=g, device=dev).bfloat16()
    kv_new = (torch.randn((wl.n_q, sp.d_latent + sp.d_rope), generator=g, device=dev)
              .bfloat16() if with_kv else None)
    seq = torch.from_numpy(wl.q_seq).to(dev)
    pos = torch.from_numpy(wl.q_pos).to(dev)
    q_out = torch.empty((wl.n_q, sp.h_index, sp.d_index), dtype=torch.uint8, device=dev)
    q_scale = torch.empty((wl.n_q, sp.h_index), dtype=torch.float32, device=dev)
    ws = api.workspace(256, dev)

    def step():
        api.quantize_index_query(qi, out=q_out, scale=q_scale)
        api.append_tokens(cache, seq, pos, k_index=k_new, kv=kv_new, ws=ws)

    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    for k in range(args.steps):
        flush_l2(flush)
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    st = api.device_status(ws)
    if st[0] != 0:
        raise RuntimeError(f"device status after input preparation: {st}")
    ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    nb = input_prep_bytes(wl, with_kv)
    hbm, _, kind = measured_peaks()
    gbs = nb / (ms / 1e3) / 1e9
    return {"ms": ms, "bytes": nb, "achieved_gbs": gbs, "frac": gbs / hbm, "peak_kind": kind,
            "launches": 2, "appends_latent": with_kv,
            "what": "bf16 indexer query -> e4m3 + scales; one bf16 key (and latent row) "
                    "per query appended at its position"}


def serving_inputs(wl) -> dict:
    """Host arrays a serving step starts from, for the end-to-end leg: the query
    tokens' sequence, position, head weights and attention query as in the
    workload; the indexer query as the projection would hand it over (for an
    e4m3 index cache in bf16 -- the e4m3 codes times their scales, so that
    quantising it again on the device gives back the workload's query up to
    the bf16 rounding of those products -- as
    ``q_index_in``; otherwise in the cache's own format as ``q_index``); and
    each query's own token -- index key and latent row, the values already
    cached at its position -- to be appended at that position
    (``k_new``/``kv_new``, None where the pool takes no single tokens: a bf16
    index pool, or a latent cache with one scale per page)."""
    import torch
    sp = wl.spec
    out = {k: torch.from_numpy(getattr(wl, k)) for k in ("q_seq", "q_pos", "w", "q")}
    ps = sp.page_size
    rows = (wl.page_table[wl.q_seq, wl.q_pos // ps].astype(np.int64) * ps + wl.q_pos % ps)
    out["k_new"] = out["kv_new"] = None
    if sp.index_dtype == "e4m3":
        qi = torch.from_numpy(wl.q_index).view(torch.float8_e4m3fn).float()
        out["q_index_in"] = (qi * torch.from_numpy(wl.q_index_scale)[..., None]).bfloat16()
        k = torch.from_numpy(wl.k_index.reshape(-1, sp.d_index)[rows]).view(torch.float8_e4m3fn)
        k = k.float() * torch.from_numpy(wl.k_index_scale.reshape(-1)[rows])[:, None]
        out["k_new"] = k.bfloat16()
    else:
        out["q_index"] = torch.from_numpy(wl.q_index)
        if wl.q_index_scale is not None:  # MXFP8: the quantised query and its scale bytes
            out["q_index_scale"] = torch.from_numpy(wl.q_index_scale)
        if sp.index_dtype == "f32":
            out["k_new"] = torch.from_numpy(wl.k_index.reshape(-1, sp.d_index)[rows])
    if sp.kv_dtype == "f32":
        out["kv_new"] = torch.from_numpy(wl.kv.reshape(-1, sp.d_qk)[rows])
    elif sp.kv_dtype == "bf16":
        kv = torch.from_numpy(wl.kv.reshape(-1, sp.d_qk)[rows].view(np.int16))
        out["kv_new"] = kv.view(torch.bfloat16)
    elif sp.kv_tile[0] == 1:
        st, sd = sp.kv_tile
        codes = torch.from_numpy(wl.kv.reshape(-1, sp.d_latent)[rows]).view(torch.float8_e4m3fn)
        sc = wl.kv_scale.reshape(wl.num_pages, ps // st, sp.d_latent // sd)
        sc = sc[rows // ps, (rows % ps) // st]                       # [n_q, d_latent / sd]
        lat = codes.float() * torch.from_numpy(np.repeat(sc, sd, axis=1))
        rope = torch.from_numpy(wl.kv_rope.reshape(-1, sp.d_rope)[rows].view(np.int16))
        out["kv_new"] = torch.cat([lat.bfloat16(), rope.view(torch.bfloat16)], dim=1)
    ins = [t for t in (out["k_new"], out["kv_new"]) if t is not None]
    if len({t.dtype for t in ins}) > 1:  # the append takes one input dtype
        out["k_new"] = out["k_new"].to(out["kv_new"].dtype)
    return out


def serving_bytes(inp: dict) -> int:
    """Host -> device bytes of one serving step's inputs."""
    return sum(v.numel() * v.element_size() for v in inp.values() if v is not None)


def measure_decode(args, wl, dev, dist=None):
    """Device-timed fused decode on one workload: the timed steps (L2 flushed
    before each), then the same steps again with events between the phases.
    Returns the step time, phase times, launches, clocks and the accounting."""
    import torch
    from indexed_sparse_attention_lightning_b200 import _abi, api
    sp = wl.spec
    cache, queries = api.upload(wl, dev)
    K = sp.top_k
    odt = "f32" if sp.kv_dtype == "f32" else "bf16"
    ws = api.workspace(api.workspace_size(cache, queries, K, _abi.SA_WS_DECODE), dev)
    idx = torch.empty((wl.n_q, K), dtype=torch.int32, device=dev)
    out, lse = api._outputs(queries, sp.d_latent, None, None, odt)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(events=None):
        api.decode(cache, queries, K, out=out, lse=lse, idx=idx, out_dtype=odt, ws=ws,
                   phase_events=events)

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    st = api.device_status(ws)
    if st[0] != _abi.SA_OK:
        raise RuntimeError(f"{sp.name}: device status after warm-up: {st}")
    idx_host = idx.cpu().numpy()
    nbytes = algorithmic_bytes(wl, idx_host)

    n_phase = len(_abi.DECODE_PHASES)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_phase + 1)]
          for _ in range(args.steps)]
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = _abi.lib().sa_kernel_launches()
    with ClockSampler(dev.index or 0) as clocks:
        for k in range(args.steps):
            flush_l2(flush)
            outer[k][0].record(stream)
            step()
            outer[k][1].record(stream)
        torch.cuda.synchronize()
    launches = _abi.lib().sa_kernel_launches() - launches0
    # Phase attribution: the same steps again with events between the phases
    # (an event between two kernels stops the next one from launching early,
    # so these steps run a little slower than the timed ones above).
    for k in range(args.steps):
        flush_l2(flush)
        step(ev[k])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = sum(a.elapsed_time(b) for a, b in outer)
    phase_ms = [sum(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(args.steps)) / args.steps
                for i in range(n_phase)]
    st = api.device_status(ws)
    if st[0] != _abi.SA_OK:
        raise RuntimeError(f"{sp.name}: device status after timing: {st}")
    return {"total_ms": total_ms, "phase_ms": phase_ms, "launches": int(launches),
            "clocks": clocks.summary(), "nbytes": nbytes, "idx_host": idx_host,
            "cache": cache, "queries": queries, "ws": ws, "idx": idx, "out": out, "lse": lse,
            "flush": flush, "odt": odt}


def summarise(wl, m: dict, n_q_all: float, total_ms: float, steps: int) -> dict:
    """The per-workload figures of a bench line."""
    from indexed_sparse_attention_lightning_b200 import _abi
    ms_per_step = total_ms / steps
    peak, _, _ = measured_peaks()
    phase_ms = m["phase_ms"]
    dom = int(np.argmax(phase_ms))
    dom_name = _abi.DECODE_PHASES[dom]
    roof = roofline(wl, dom_name, phase_ms[dom], m["nbytes"],
                    algorithmic_flops(wl, m["idx_host"]))
    step_gbs = m["nbytes"]["total"] / (ms_per_step / 1e3) / 1e9
    return {
        "value": n_q_all * steps / (total_ms / 1e3), "ms_per_step": ms_per_step,
        "roofline": roof,
        "path_hbm": {"bytes_per_step": m["nbytes"]["total"], "achieved_gbs": step_gbs,
                     "frac_of_measured": step_gbs / peak, "frac_of_8tbs": step_gbs / SPEC_HBM_GBS},
        "phases_ms": dict(zip(_abi.DECODE_PHASES, phase_ms)),
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
    }


def time_e2e(args, wl, m: dict, dev):
    """End to end through the public API with host buffers: every step copies
    its inputs from pinned host memory -- the bf16 indexer query, head weights,
    attention query, sequence and position of each query, and each query's own
    new token -- then quantises the indexer query, appends the new tokens to
    the paged caches and decodes (all on the device), and reads the output and
    lse back.  Steps are pipelined the way a serving loop runs them -- the
    copies of one step overlap the compute of its neighbours (copy-in stream,
    compute stream, copy-out stream; inputs and outputs double-buffered) -- and
    the time runs from the first copy-in to the last copy-out.  No L2 flush
    runs inside this loop: a serving loop has none."""
    import torch
    from indexed_sparse_attention_lightning_b200 import api
    sp = wl.spec
    cache, queries, ws, idx = m["cache"], m["queries"], m["ws"], m["idx"]
    out, lse, odt = m["out"], m["lse"], m["odt"]
    host = {k: (v.pin_memory() if v is not None else None)
            for k, v in serving_inputs(wl).items()}
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def dev_set():
        d = {k: (torch.empty_like(v, device=dev) if v is not None else None)
             for k, v in host.items()}
        q = dataclasses.replace(
            queries, q_seq=d["q_seq"], q_pos=d["q_pos"], w=d["w"], q=d["q"],
            q_index=d.get("q_index", torch.empty_like(queries.q_index)),
            q_index_scale=d.get("q_index_scale",
                                None if queries.q_index_scale is None
                                else torch.empty_like(queries.q_index_scale)))
        return d, q

    bufs = [dev_set(), dev_set()]
    obuf = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
    hout = [(torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
             torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)) for _ in range(2)]
    aws = api.workspace(256, dev)

    def pipelined(n):
        if n <= 0:
            return 0.0
        in_done = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        out_done = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for k in range(n):
            b = k % 2
            d, q = bufs[b]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp_done[k - 2])  # buffer b no longer read
                for key, v in host.items():
                    if v is not None:
                        d[key].copy_(v, non_blocking=True)
                in_done[k].record(s_in)
            comp.wait_event(in_done[k])
            if k >= 2:
                comp.wait_event(out_done[k - 2])  # output b has been read back
            if "q_index_in" in d:
                api.quantize_index_query(d["q_index_in"], out=q.q_index,
                                         scale=q.q_index_scale)
            if d["k_new"] is not None or d["kv_new"] is not None:
                api.append_tokens(cache, d["q_seq"], d["q_pos"], k_index=d["k_new"],
                                  kv=d["kv_new"], ws=aws)
            api.decode(cache, q, sp.top_k, out=obuf[b][0], lse=obuf[b][1], idx=idx,
                       out_dtype=odt, ws=ws)
            comp_done[k].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[k])
                hout[b][0].copy_(obuf[b][0], non_blocking=True)
                hout[b][1].copy_(obuf[b][1], non_blocking=True)
                out_done[k].record(s_out)
        s_out.wait_event(out_done[n - 1])
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    pipelined(args.warmup)
    total = pipelined(args.steps)
    st = api.device_status(aws)
    if st[0] != 0:
        raise RuntimeError(f"device status after the end-to-end appends: {st}")
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
    return {"ms_per_step": total / args.steps, "h2d": serving_bytes(host), "d2h": d2h,
            "appends_keys": host["k_new"] is not None,
            "appends_latent": host["kv_new"] is not None}


def other_workloads(args, dev) -> dict:
    """The other configurations, each timed like the headline in the same run
    (device time, L2 flushed before every step; no end-to-end or CPU leg)."""
    import torch
    from indexed_sparse_attention_lightning_b200 import workloads as W
    res = {}
    for sp in W.CONFIGS:
        if sp.name == args.workload:
            continue
        wl = W.make_workload(sp)
        m = measure_decode(args, wl, dev)
        r = summarise(wl, m, wl.n_q, m["total_ms"], args.steps)
        r["config"] = workload_config(sp, wl, 1)
        res[sp.name] = r
        del m, wl
        torch.cuda.empty_cache()
    return res


def run_ours(args, rank: int, world: int, dist):
    import torch
    from indexed_sparse_attention_lightning_b200 import workloads as W

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sp = rank_spec(W.spec(args.workload), rank)
    wl = W.make_workload(sp)
    m = measure_decode(args, wl, dev, dist)
    e2e = None if args.no_e2e else time_e2e(args, wl, m, dev)
    prep = time_input_prep(args, wl, m["cache"], dev, m["flush"])
    total_ms, e2e_step_ms, n_q_all = reduce_over_ranks(
        dist, dev, m["total_ms"], e2e["ms_per_step"] if e2e else 0.0, wl.n_q)
    extra = None
    if world == 1 and not args.no_extra:
        del m["cache"], m["queries"], m["ws"], m["out"], m["lse"], m["idx"], m["flush"]
        torch.cuda.empty_cache()
        extra = other_workloads(args, dev)
    if rank != 0:
        return 0

    summ = summarise(wl, m, n_q_all, total_ms, args.steps)
    roof = summ["roofline"]
    dom_name = roof["kernel"]
    csrc = "indexed_sparse_attention_lightning_b200/csrc/"
    shared = [csrc + f for f in ("common.cuh", "sm100.cuh", "internal.h")]
    kernel_src = {"indexer": [csrc + "indexer_mma.cu", csrc + "plan.cu"] + shared,
                  "topk": [csrc + "topk.cu"] + shared,
                  "attention": [csrc + "sfa_mma.cu"] + shared}
    traffic = traffic_for(dom_name, kernel_src[dom_name], sp.name)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n, spent = time_oracle(wl, args.cpu_seconds)
        import oracle
        cpu = {"value": n / spent, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
               "sample": f"{n} of {wl.n_q} queries of the same workload (fp64 oracle: scores, "
                         f"top-K, attention), {spent:.1f} s"}

    line = {
        "metric": METRIC, "value": summ["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": summ["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"{sp.index_dtype}+{sp.kv_dtype}", "data": "synthetic",
        "config": workload_config(sp, wl, world),
        "roofline": dict(roof, traffic=traffic if roof["bound"] == "hbm" else None),
        "path_hbm": summ["path_hbm"],
        "phases_ms": summ["phases_ms"],
        "gpu_launches": summ["gpu_launches"],
        "clocks": summ["clocks"],
        "cpu_baseline": cpu,
        "input_prep": prep,
    }
    if e2e:
        line["e2e"] = {"value": n_q_all / (e2e_step_ms / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "what": "pinned host inputs -> quantise the indexer query, append each "
                               "query's new token (index key: %s, latent row: %s), decode -> "
                               "output and lse to the host; pipelined over three streams"
                               % ("yes" if e2e["appends_keys"] else "no",
                                  "yes" if e2e["appends_latent"] else "no")}
    if extra is not None:
        line["other_configs"] = extra
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        return run_reference(args, rank, world)   # rank 0 only; no process group needed
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        # short enough that ranks waiting on a lost peer fail instead of hanging,
        # long enough for every rank to draw its inputs before the first barrier
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
