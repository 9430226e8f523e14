#!/usr/bin/env python3
"""Sparse-attention decode throughput on B200: indexer + top-K + sparse MLA attention.

One step = one fused ``sa_decode`` over one batch of synthetic queries (all
three steps of the path).  Prints ONE JSON line (rank 0):

  value     query-tokens/s over all ranks, device time (CUDA events), inputs
            resident in HBM, L2 flushed before every timed step (a 256 MiB
            buffer written, then read back, outside the timed region);
  e2e       the same metric through the public API with host buffers: pinned
            host -> device copy of the step's queries, the call, device -> host
            copy of the outputs, all inside the timed region (there the 256 MiB
            write that flushes L2 sits inside the timed region too);
  roofline  the dominant phase's algorithmic bytes / its event-timed duration
            against the measured HBM copy bandwidth;
  cpu_baseline  the fp64 oracle on a bounded sample, on this host's cores.

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
    key_b = sp.d_index * {"e4m3": 1, "bf16": 2, "f32": 4}[sp.index_dtype]
    scale_b = 4 if sp.index_dtype == "e4m3" else 0
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


def run_ours(args, rank: int, world: int, dist):
    import torch
    from indexed_sparse_attention_lightning_b200 import _abi, api
    from indexed_sparse_attention_lightning_b200 import workloads as W

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sp = rank_spec(W.spec(args.workload), rank)
    wl = W.make_workload(sp)
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
        raise RuntimeError(f"device status after warm-up: {st}")
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
    with ClockSampler(local) as clocks:
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
        raise RuntimeError(f"device status after timing: {st}")

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory and reads its output back.  Steps are
    # pipelined the way a serving loop runs them -- the copies of one step
    # overlap the compute of its neighbours (copy-in stream, compute stream,
    # copy-out stream; inputs and outputs double-buffered) -- and the time
    # runs from the first copy-in to the last copy-out.
    e2e = None
    if not args.no_e2e:
        import dataclasses as _dc
        host_in = api.host_queries(wl, pin=True)
        comp = stream
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        qbuf = [queries, _dc.replace(queries, **{k: torch.empty_like(v)
                                                 for k, v in queries.tensors().items()
                                                 if v is not None})]
        obuf = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
        hout = [(torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
                 torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)) for _ in range(2)]

        def pipelined(n):
            if n <= 0:
                return 0.0, 0
            in_done = [torch.cuda.Event() for _ in range(n)]
            comp_done = [torch.cuda.Event() for _ in range(n)]
            out_done = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            h2d = 0
            t0.record(s_in)
            for k in range(n):
                b = k % 2
                with torch.cuda.stream(s_in):
                    if k >= 2:
                        s_in.wait_event(comp_done[k - 2])  # buffer b no longer read
                    h2d = qbuf[b].copy_from(host_in, non_blocking=True)
                    in_done[k].record(s_in)
                comp.wait_event(in_done[k])
                if k >= 2:
                    comp.wait_event(out_done[k - 2])  # output b has been read back
                flush.zero_()
                api.decode(cache, qbuf[b], K, out=obuf[b][0], lse=obuf[b][1], idx=idx,
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
            return t0.elapsed_time(t1), h2d

        pipelined(args.warmup)
        e2e_total, h2d = pipelined(args.steps)
        d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
        e2e = {"ms_per_step": e2e_total / args.steps, "h2d": h2d, "d2h": d2h}

    prep = time_input_prep(args, wl, cache, dev, flush)

    total_ms, e2e_step_ms, n_q_all = reduce_over_ranks(
        dist, dev, total_ms, e2e["ms_per_step"] if e2e else 0.0, wl.n_q)
    if rank != 0:
        return 0

    ms_per_step = total_ms / args.steps
    value = n_q_all * args.steps / (total_ms / 1e3)
    peak, _, peak_kind = measured_peaks()
    dom = int(np.argmax(phase_ms))
    dom_name = _abi.DECODE_PHASES[dom]
    roof = roofline(wl, dom_name, phase_ms[dom], nbytes, algorithmic_flops(wl, idx_host))
    step_gbs = nbytes["total"] / (ms_per_step / 1e3) / 1e9
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
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": f"{sp.index_dtype}+{sp.kv_dtype}", "data": "synthetic",
        "config": workload_config(sp, wl, world),
        "roofline": dict(roof, traffic=traffic if roof["bound"] == "hbm" else None),
        "path_hbm": {"bytes_per_step": nbytes["total"], "achieved_gbs": step_gbs,
                     "frac_of_measured": step_gbs / peak, "frac_of_8tbs": step_gbs / SPEC_HBM_GBS},
        "phases_ms": dict(zip(_abi.DECODE_PHASES, phase_ms)),
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
        "input_prep": prep,
    }
    if e2e:
        line["e2e"] = {"value": n_q_all / (e2e_step_ms / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]}
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
