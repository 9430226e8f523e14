"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (runs without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

from indexed_sparse_attention_lightning_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sa.h")).read()
    return sorted(set(re.findall(r"SA_API\s+[\w\s\*]*?\b(sa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 8
    assert sorted(_abi.EXPORTS) == names
    for n in names:
        assert hasattr(L, n), n
    assert L.sa_version() >= 100


def test_status_strings(L):
    for s in range(7):
        assert _abi.status_string(s)
    assert _abi.status_string(99) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned non-null stand-in; never dereferenced


def good_cache(**kw):
    c = _abi.SaCache(page_table=FAKE, seq_len=FAKE, batch=2, max_pages=4, num_pages=8,
                     page_size=64, index_dtype=_abi.SA_E4M3, k_index=FAKE, k_index_scale=FAKE,
                     d_index=128, kv_dtype=_abi.SA_BF16, kv=FAKE, kv_rope=None, kv_scale=None,
                     d_latent=512, d_rope=64)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def good_query(**kw):
    q = _abi.SaQuery(n_q=2, q_seq=FAKE, q_pos=FAKE, max_visible=256, q_index=FAKE,
                     q_index_scale=FAKE, w=FAKE, h_index=64, q_dtype=_abi.SA_BF16, q=FAKE,
                     heads=128, sm_scale=0.0416)
    for k, v in kw.items():
        setattr(q, k, v)
    return q


def ws_size(L, c, q, k=2048, uses=_abi.SA_WS_DECODE):
    return L.sa_workspace_size(ctypes.byref(c), ctypes.byref(q), k, uses)


def test_workspace_size_valid_and_invalid(L):
    n = ws_size(L, good_cache(), good_query())
    # status + scores [2, 256] + idx [2, 2048], 256-byte aligned pieces
    assert n >= 256 + 2 * 256 * 4 + 2 * 2048 * 4 and n % 256 == 0
    assert ws_size(L, good_cache(page_size=32), good_query()) == 0
    assert ws_size(L, good_cache(d_index=100), good_query()) == 0
    assert ws_size(L, good_cache(), good_query(max_visible=4 * 64 + 1)) == 0
    assert ws_size(L, good_cache(), good_query(), k=0) == 0
    assert ws_size(L, good_cache(kv_dtype=_abi.SA_E4M3), good_query()) == 0  # no scales
    assert ws_size(L, good_cache(), good_query(q_index_scale=None)) == 0


FP8_KV = {"kv_dtype": _abi.SA_E4M3, "kv_rope": FAKE, "kv_scale": FAKE}


def test_mxfp8_index_argument_checks(L):
    """MXFP8 index data (one E8M0 byte per 32 values) needs both scale arrays,
    16-byte aligned, and a dimension that is a whole number of groups; it names
    index data only, and no key encoder exists for appending to such a pool."""
    mx = {"index_dtype": _abi.SA_MXFP8}
    assert ws_size(L, good_cache(**mx), good_query()) > 0
    assert ws_size(L, good_cache(**mx, d_index=48), good_query()) == 0     # 1.5 groups
    assert ws_size(L, good_cache(**mx, k_index_scale=None), good_query()) == 0
    assert ws_size(L, good_cache(**mx), good_query(q_index_scale=None)) == 0
    assert ws_size(L, good_cache(**mx), good_query(q_index_scale=FAKE + 4)) == 0
    assert decode_call(L, good_cache(kv_dtype=_abi.SA_MXFP8), good_query()) == \
        _abi.SA_ERR_UNSUPPORTED
    t = new_tokens()
    assert L.sa_append_tokens(ctypes.byref(good_cache(**mx)), ctypes.byref(t), FAKE, 1 << 20,
                              None) == _abi.SA_ERR_UNSUPPORTED


@pytest.mark.parametrize("tile,ok", [
    ((0, 0), True),       # one scale per page
    ((1, 128), True),     # per token and 128 latent dims
    ((64, 512), True), ((4, 16), True),
    ((3, 128), False),    # does not divide the page
    ((1, 100), False),    # does not divide the latent dims
    ((1, 8), False),      # not a multiple of 16 dims
    ((-1, 128), False), ((1, 0), False),
])
def test_fp8_scale_tile_validation(L, tile, ok):
    c = good_cache(**FP8_KV, kv_scale_tokens=tile[0], kv_scale_dims=tile[1])
    assert (ws_size(L, c, good_query()) > 0) == ok


def decode_call(L, c, q, k=2048, ws=FAKE, ws_bytes=1 << 30, out=FAKE):
    return L.sa_decode(ctypes.byref(c), ctypes.byref(q), k, None, out, _abi.SA_BF16, None, ws,
                       ws_bytes, None)


@pytest.mark.parametrize("mutation,expect", [
    ({"cache": {"page_table": None}}, _abi.SA_ERR_INVALID_ARG),
    ({"cache": {"kv": FAKE + 4}}, _abi.SA_ERR_INVALID_ARG),          # misaligned
    ({"cache": {"page_size": 16}}, _abi.SA_ERR_UNSUPPORTED),
    ({"cache": {"index_dtype": 7}}, _abi.SA_ERR_UNSUPPORTED),
    ({"cache": {"kv_dtype": 7}}, _abi.SA_ERR_UNSUPPORTED),
    ({"cache": {"num_pages": 0}}, _abi.SA_ERR_INVALID_ARG),
    ({"query": {"n_q": -1}}, _abi.SA_ERR_INVALID_ARG),
    ({"query": {"n_q": 70000}}, _abi.SA_ERR_UNSUPPORTED),
    ({"query": {"w": None}}, _abi.SA_ERR_INVALID_ARG),
    ({"query": {"q_dtype": _abi.SA_E4M3}}, _abi.SA_ERR_UNSUPPORTED),
    ({"query": {"sm_scale": float("nan")}}, _abi.SA_ERR_INVALID_ARG),
    ({"k": 0}, _abi.SA_ERR_INVALID_ARG),
    ({"ws": None}, _abi.SA_ERR_WORKSPACE),
    ({"ws_bytes": 16}, _abi.SA_ERR_WORKSPACE),
    ({"ws": FAKE + 16}, _abi.SA_ERR_WORKSPACE),                      # not 256-aligned
    ({"out": None}, _abi.SA_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments_before_launch(L, mutation, expect):
    c = good_cache(**mutation.get("cache", {}))
    q = good_query(**mutation.get("query", {}))
    kw = {k: v for k, v in mutation.items() if k in ("k", "ws", "ws_bytes", "out")}
    assert decode_call(L, c, q, **kw) == expect


def test_other_entry_points_reject_bad_arguments(L):
    c, q = good_cache(), good_query()
    # scores leading dimension smaller than the visible range
    assert L.sa_indexer_score(ctypes.byref(c), ctypes.byref(q), FAKE, 100, FAKE, 1 << 20,
                              None) == _abi.SA_ERR_INVALID_ARG
    assert L.sa_topk(FAKE, 10, FAKE, 2, 20, 4, FAKE, FAKE, 1 << 20, None) == \
        _abi.SA_ERR_INVALID_ARG
    assert L.sa_topk(FAKE, 10, FAKE, 2, 10, 0, FAKE, FAKE, 1 << 20, None) == \
        _abi.SA_ERR_INVALID_ARG
    assert L.sa_topk(FAKE, 10, FAKE, 2, 10, 4, FAKE, None, 0, None) == _abi.SA_ERR_WORKSPACE
    assert L.sa_sparse_mla_attn(ctypes.byref(c), ctypes.byref(q), None, 2048, FAKE,
                                _abi.SA_BF16, None, FAKE, 1 << 20, None) == \
        _abi.SA_ERR_INVALID_ARG
    assert L.sa_sparse_mla_attn(ctypes.byref(c), ctypes.byref(q), FAKE, 2048, FAKE,
                                _abi.SA_E4M3, None, FAKE, 1 << 20, None) == \
        _abi.SA_ERR_UNSUPPORTED
    assert L.sa_device_status(None, 0, None, None) == _abi.SA_ERR_WORKSPACE


def test_quantize_index_query_checks_arguments_before_launch(L):
    q = L.sa_quantize_index_query
    assert q(FAKE, _abi.SA_BF16, -1, 64, 128, FAKE, FAKE, None) == _abi.SA_ERR_INVALID_ARG
    assert q(FAKE, _abi.SA_BF16, 4, 0, 128, FAKE, FAKE, None) == _abi.SA_ERR_INVALID_ARG
    assert q(FAKE, _abi.SA_E4M3, 4, 64, 128, FAKE, FAKE, None) == _abi.SA_ERR_UNSUPPORTED
    assert q(None, _abi.SA_BF16, 4, 64, 128, FAKE, FAKE, None) == _abi.SA_ERR_INVALID_ARG
    assert q(FAKE + 8, _abi.SA_F32, 4, 64, 128, FAKE, FAKE, None) == _abi.SA_ERR_INVALID_ARG
    assert q(FAKE, _abi.SA_BF16, 0, 64, 128, None, None, None) == _abi.SA_OK  # nothing to do


def new_tokens(**kw):
    t = _abi.SaNewTokens(n_new=2, seq=FAKE, pos=FAKE, in_dtype=_abi.SA_BF16, k_index=FAKE,
                         kv=FAKE)
    for k, v in kw.items():
        setattr(t, k, v)
    return t


@pytest.mark.parametrize("cache,tokens,ws,expect", [
    ({"page_table": None}, {}, FAKE, _abi.SA_ERR_INVALID_ARG),
    ({}, {"n_new": -1}, FAKE, _abi.SA_ERR_INVALID_ARG),
    ({}, {"in_dtype": _abi.SA_E4M3}, FAKE, _abi.SA_ERR_UNSUPPORTED),
    ({}, {"seq": None}, FAKE, _abi.SA_ERR_INVALID_ARG),
    ({}, {"kv": FAKE + 2}, FAKE, _abi.SA_ERR_INVALID_ARG),            # misaligned input
    ({}, {}, None, _abi.SA_ERR_WORKSPACE),
    ({}, {}, FAKE + 64, _abi.SA_ERR_WORKSPACE),                        # not 256-aligned
    # e4m3 latent: only one-token scale tiles can take a new token
    ({**FP8_KV}, {}, FAKE, _abi.SA_ERR_UNSUPPORTED),
    ({**FP8_KV, "kv_scale_tokens": 16, "kv_scale_dims": 128}, {}, FAKE,
     _abi.SA_ERR_UNSUPPORTED),
])
def test_append_tokens_checks_arguments_before_launch(L, cache, tokens, ws, expect):
    c, t = good_cache(**cache), new_tokens(**tokens)
    assert L.sa_append_tokens(ctypes.byref(c), ctypes.byref(t), ws, 1 << 20, None) == expect
    if tokens == {"n_new": -1}:
        assert L.sa_append_tokens(ctypes.byref(c), None, FAKE, 1 << 20, None) == \
            _abi.SA_ERR_INVALID_ARG


def test_append_workspace_needs_no_query(L):
    c = good_cache()
    assert L.sa_workspace_size(ctypes.byref(c), None, 0, _abi.SA_WS_APPEND) == 256
    assert L.sa_workspace_size(ctypes.byref(good_cache(page_size=16)), None, 0,
                               _abi.SA_WS_APPEND) == 0


def test_struct_layout_matches_the_header(tmp_path):
    """The ctypes mirrors have the same size and field offsets as the C structs
    of include/sa.h, as gcc lays them out."""
    structs = {"sa_cache": _abi.SaCache, "sa_query": _abi.SaQuery,
               "sa_new_tokens": _abi.SaNewTokens}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "sa.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'    printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'    printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ['    return 0;', '}']
    src = tmp_path / "layout.c"
    exe = tmp_path / "layout"
    src.write_text("\n".join(lines) + "\n")
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "include")
    import subprocess
    subprocess.run(["gcc", "-std=c11", "-I", include, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    seen = {}
    for line in out.splitlines():
        cname, field, value = line.split()
        seen[(cname, field)] = int(value)
    for cname, py in structs.items():
        assert seen[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert seen[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


class _OnDevice(torch.Tensor):
    """A host tensor that reports itself as a CUDA tensor, to exercise the
    binding's dtype, shape and layout checks without a GPU (never passed on)."""

    @property
    def is_cuda(self):
        return True


def test_binding_refuses_tensors_it_would_misread():
    from indexed_sparse_attention_lightning_b200 import api
    need = api._need
    with pytest.raises(_abi.SaError, match="CUDA tensor"):
        need(torch.zeros(4, dtype=torch.int32), "seq", torch.int32)
    dev = lambda t: t.as_subclass(_OnDevice)  # noqa: E731
    need(dev(torch.zeros(4, dtype=torch.int32)), "seq", torch.int32, (4,))
    with pytest.raises(_abi.SaError, match="dtype"):
        need(dev(torch.zeros(4, dtype=torch.int64)), "seq", torch.int32)
    with pytest.raises(_abi.SaError, match="shape"):
        need(dev(torch.zeros(5, dtype=torch.int32)), "seq", torch.int32, (4,))
    with pytest.raises(_abi.SaError, match="contiguous"):
        need(dev(torch.zeros((4, 6), dtype=torch.float32)[:, ::2]), "x")
    with pytest.raises(_abi.SaError, match="required"):
        need(None, "x")
    need(None, "x", optional=True)
    # score matrices may have padded rows but need unit column stride
    api._need_rows(dev(torch.zeros((3, 10), dtype=torch.float32)[:, :7]), "scores", 3, 7)
    with pytest.raises(_abi.SaError):
        api._need_rows(dev(torch.zeros((3, 10), dtype=torch.float32)[:, ::2]), "scores", 3, 5)
    with pytest.raises(_abi.SaError):
        api._need_rows(dev(torch.zeros((3, 10), dtype=torch.float32)), "scores", 3, 11)
    # the entry points check before they reach the library
    with pytest.raises(_abi.SaError, match="CUDA tensor"):
        api.quantize_index_query(torch.zeros((2, 64, 128), dtype=torch.bfloat16))
