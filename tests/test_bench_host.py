"""Host-side accounting of bench.py: algorithmic bytes and flops per phase and
the choice of roofline (decode against HBM, chunked prefill against the
tensor pipe).  No GPU: the selections are made up on the host."""
import numpy as np

import bench
from indexed_sparse_attention_lightning_b200 import workloads as W


def _first_k(wl, K):
    """Positions 0 .. min(K, V_t) - 1 of every query, -1 padded."""
    idx = np.full((wl.n_q, K), -1, dtype=np.int32)
    for t, v in enumerate(wl.visible):
        n = min(K, int(v))
        idx[t, :n] = np.arange(n)
    return idx


def test_decode_bytes_and_hbm_roofline():
    wl = W.make_workload(W.spec("tiny_decode_b1_1k_fp32"))
    sp = wl.spec
    idx = _first_k(wl, sp.top_k)
    nb = bench.algorithmic_bytes(wl, idx)
    V = int(wl.visible.sum())
    assert nb["indexer"] == V * sp.d_index * 4                     # fp32 keys, no scales
    rows = int(np.minimum(wl.visible, sp.top_k).sum()) * (sp.d_latent + sp.d_rope) * 4
    outs = wl.n_q * sp.heads * (sp.d_latent * 4 + 4)
    assert nb["attention"] == rows + outs
    assert nb["total"] == nb["indexer"] + nb["attention"]
    r = bench.roofline(wl, "attention", 1.0, nb, bench.algorithmic_flops(wl, idx))
    hbm, _, _ = bench.measured_peaks()
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert np.isclose(r["achieved"], nb["attention"] / 1e-3 / 1e9)
    assert np.isclose(r["frac"], r["achieved"] / hbm)


def test_fp8_cache_counts_each_scale_tile_once():
    import dataclasses
    sp = dataclasses.replace(W.spec("decode_b8_8k"), batch=1, seq_len=("fixed", 256),
                             kv_dtype="e4m3", kv_scale_tile=(1, 128), top_k=64)
    wl = W.make_workload(sp)
    idx = _first_k(wl, sp.top_k)
    nb = bench.algorithmic_bytes(wl, idx)
    per_row = sp.d_latent + 2 * sp.d_rope + 4 * (sp.d_latent // 128)
    assert nb["attention"] == 64 * per_row + sp.heads * (sp.d_latent * 2 + 4)


def test_prefill_is_reported_against_the_tensor_pipe():
    import dataclasses
    sp = dataclasses.replace(W.spec("prefill_4096q_64k"), seq_len=("fixed", 4096),
                             queries=("prefill", 4032, 64))
    wl = W.make_workload(sp)
    assert wl.n_q > wl.seq_len.shape[0]
    idx = _first_k(wl, sp.top_k)
    fl = bench.algorithmic_flops(wl, idx)
    assert fl["indexer"] == int(wl.visible.sum()) * 2 * sp.h_index * sp.d_index
    assert fl["attention"] == int((idx >= 0).sum()) * 2 * sp.heads * (2 * sp.d_latent + sp.d_rope)
    _, bf16, _ = bench.measured_peaks()
    r = bench.roofline(wl, "indexer", 2.0, bench.algorithmic_bytes(wl, idx), fl)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert np.isclose(r["peak"], 2 * bf16)                          # e4m3 indexer
    assert np.isclose(r["achieved"], fl["indexer"] / 2e-3 / 1e12)
    r = bench.roofline(wl, "attention", 2.0, bench.algorithmic_bytes(wl, idx), fl)
    assert np.isclose(r["peak"], bf16)


def test_input_prep_bytes():
    import dataclasses
    sp = dataclasses.replace(W.spec("decode_b8_8k"), batch=2, seq_len=("fixed", 128))
    wl = W.make_workload(sp)
    n, h, d, D = wl.n_q, sp.h_index, sp.d_index, sp.d_latent + sp.d_rope
    q = n * h * d * 3 + n * h * 4
    keys = n * (3 * d + 4)
    assert bench.input_prep_bytes(wl, False) == q + keys
    assert bench.input_prep_bytes(wl, True) == q + keys + n * (D * 2 + D * 2)
    sp8 = dataclasses.replace(sp, kv_dtype="e4m3", kv_scale_tile=(1, 128))
    wl8 = W.make_workload(sp8)
    stored = sp.d_latent + 2 * sp.d_rope + 4 * (sp.d_latent // 128)
    assert bench.input_prep_bytes(wl8, True) == q + keys + n * (D * 2 + stored)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the same metric and workload config as the GPU arm."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_decode_b1_1k_fp32", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, check=True)
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    wl = W.make_workload(W.spec("tiny_decode_b1_1k_fp32"))
    ours = bench.workload_config(wl.spec, wl, 1)
    assert {k: v for k, v in d["config"].items() if k not in ("l2", "sample")} == \
        {k: v for k, v in ours.items() if k != "l2"}


def test_end_to_end_copy_accounting():
    """The end-to-end leg copies every query input of a step and counts its bytes:
    the count equals the bytes of the workload's query arrays, and the copy
    lands them bit for bit (host buffers standing in for the device here)."""
    import dataclasses
    import torch
    from indexed_sparse_attention_lightning_b200 import api
    wl = W.make_workload(dataclasses.replace(W.spec("decode_b8_8k"), batch=3,
                                             seq_len=("fixed", 300)))
    host = api.host_queries(wl, pin=False)
    want = sum(getattr(wl, k).nbytes for k in ("q_seq", "q_pos", "q_index", "q_index_scale",
                                               "w", "q"))
    _, queries = api.upload(wl, "cpu")
    dst = dataclasses.replace(queries, **{k: torch.zeros_like(v)
                                          for k, v in queries.tensors().items() if v is not None})
    assert dst.copy_from(host, non_blocking=False) == want
    for k, v in queries.tensors().items():
        if v is not None:
            assert torch.equal(getattr(dst, k), v), k


def test_serving_inputs_are_the_cached_tokens_and_their_bytes_are_counted():
    """The end-to-end leg's host inputs: each query's new token is the row
    already cached at its position (so appending it keeps the cache), the
    indexer query is handed over in bf16 for the e4m3 cache, and the bytes
    copied per step are exactly those of the arrays."""
    import dataclasses
    import torch
    wl = W.make_workload(dataclasses.replace(W.spec("decode_b8_8k"), batch=3,
                                             seq_len=("list", (300, 77, 129))))
    inp = bench.serving_inputs(wl)
    sp = wl.spec
    rows = wl.page_table[wl.q_seq, wl.q_pos // 64].astype(np.int64) * 64 + wl.q_pos % 64
    kv = wl.kv.reshape(-1, sp.d_qk)[rows]
    assert np.array_equal(inp["kv_new"].view(torch.int16).numpy().view(np.uint16), kv)
    k = torch.from_numpy(wl.k_index.reshape(-1, sp.d_index)[rows]).view(torch.float8_e4m3fn)
    want = (k.float() * torch.from_numpy(wl.k_index_scale.reshape(-1)[rows])[:, None]).bfloat16()
    assert torch.equal(inp["k_new"], want)
    assert inp["q_index_in"].dtype == torch.bfloat16
    assert inp["q_index_in"].shape == (wl.n_q, sp.h_index, sp.d_index)
    n = sum(a.nbytes for a in (wl.q_seq, wl.q_pos, wl.w, wl.q))
    n += wl.n_q * (sp.h_index * sp.d_index + sp.d_index + sp.d_qk) * 2
    assert bench.serving_bytes(inp) == n
    # a latent cache with one scale per page takes no single tokens
    wl8 = W.make_workload(dataclasses.replace(W.spec("decode_b2_1m_fp8kv_clustered"), batch=1,
                                              seq_len=("fixed", 70000)))
    assert bench.serving_inputs(wl8)["kv_new"] is None
