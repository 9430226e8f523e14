"""sa_decode_noalloc: the fused decode for callers that cannot allocate device
memory (code running under a host that owns every device allocation, or loops
where a cudaMalloc is not allowed).  Its scratch is a static device array of
the library, so it must give the same results as sa_decode with a caller
workspace -- on repeated calls, since the array keeps the previous call's
contents -- and must refuse requests larger than that array.

Collected last on purpose; it passes on its own in a fresh process as well as
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from indexed_sparse_attention_lightning_b200 import _abi, api
from indexed_sparse_attention_lightning_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _noalloc(cache, queries, top_k, idx, out, lse):
    c, q = cache.struct(), queries.struct()
    st = _abi.lib().sa_decode_noalloc(ctypes.byref(c), ctypes.byref(q), top_k, idx.data_ptr(),
                                      out.data_ptr(), _abi.SA_BF16, lse.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_workspace_decode_on_consecutive_calls():
    wl = W.make_workload(W.DECODE_B8_8K)
    K = wl.spec.top_k
    cache, queries = api.upload(wl)
    ws = api.workspace(api.workspace_size(cache, queries, K, _abi.SA_WS_DECODE))
    assert ws.numel() <= _abi.NOALLOC_SCRATCH_BYTES
    ref_idx = torch.empty((wl.n_q, K), dtype=torch.int32, device="cuda")
    ref_out, ref_lse, _ = api.decode(cache, queries, K, idx=ref_idx, ws=ws)
    assert api.device_status(ws) == (_abi.SA_OK, 0)
    ref_out = ref_out.float().cpu().numpy()
    for _ in range(2):
        idx = torch.full((wl.n_q, K), -9, dtype=torch.int32, device="cuda")
        out = torch.full_like(api._outputs(queries, wl.spec.d_latent, None, None, "bf16")[0],
                              float("nan"))
        lse = torch.full((wl.n_q, wl.spec.heads), float("nan"), device="cuda")
        assert _noalloc(cache, queries, K, idx, out, lse) == _abi.SA_OK
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        parity.check_attention(out.float().cpu().numpy(), ref_out, wl.spec.kv_dtype)
        parity.check_lse(lse.cpu().numpy(), ref_lse.cpu().numpy())


def _noalloc_status():
    detail = ctypes.c_int32(-1)
    st = _abi.lib().sa_noalloc_status(torch.cuda.current_stream().cuda_stream,
                                      ctypes.byref(detail))
    return st, detail.value


def test_noalloc_reports_bad_data_through_its_status_reader():
    """A bad page id (host-side input, checked by the kernels) must show up in
    the static array's status word, and a clean call must clear it again."""
    wl = W.make_workload(W.DECODE_B8_8K)
    K = wl.spec.top_k
    cache, queries = api.upload(wl)
    idx = torch.empty((wl.n_q, K), dtype=torch.int32, device="cuda")
    out, lse = api._outputs(queries, wl.spec.d_latent, None, None, "bf16")
    cache.page_table[3, 5] = wl.num_pages + 3
    assert _noalloc(cache, queries, K, idx, out, lse) == _abi.SA_OK
    assert _noalloc_status() == (_abi.SA_ERR_DEVICE_FAULT, _abi.SA_DETAIL_BAD_PAGE)
    cache.page_table[3, 5] = int(wl.page_table[3, 5])
    assert _noalloc(cache, queries, K, idx, out, lse) == _abi.SA_OK
    assert _noalloc_status() == (_abi.SA_OK, 0)


def test_noalloc_rejects_requests_beyond_its_scratch():
    wl = W.make_workload(W.DECODE_B8_8K)
    cache, queries = api.upload(wl)
    # 4096 queries over 8192 positions need 4096 * 8192 * 4 B of scores (> 32 MiB);
    # the call must refuse before launching anything.
    big = api.DeviceQueries(**{**queries.__dict__})
    c, q = cache.struct(), big.struct()
    q.n_q = 4096
    assert _abi.lib().sa_workspace_size(ctypes.byref(c), ctypes.byref(q), 2048,
                                        _abi.SA_WS_DECODE) > _abi.NOALLOC_SCRATCH_BYTES
    st = _abi.lib().sa_decode_noalloc(ctypes.byref(c), ctypes.byref(q), 2048, None, 1 << 20,
                                      _abi.SA_BF16, None, None)
    assert st == _abi.SA_ERR_WORKSPACE
