"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol that include/nsa.h declares, and rejects bad arguments with a status
code before it touches the device (no CUDA call is reached by these cases)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import sparse_long_context_nsa_b200 as nsa
from sparse_long_context_nsa_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return nsa.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "nsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_\w+)\s*\(", src)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(nsa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_has_no_torch_or_oracle_dependency(lib):
    # the .so is self-contained C ABI: it must not pull in libtorch or the oracle
    with open(nsa.LIB_PATH, "rb") as f:
        blob = f.read()
    assert b"libtorch" not in blob and b"libc10" not in blob
    assert b"oracle_compress" not in blob


def test_status_strings(lib):
    names = [nsa.nsa_status_string(i) for i in range(6)]
    assert names == ["NSA_OK", "NSA_ERR_INVALID_ARG", "NSA_ERR_UNSUPPORTED", "NSA_ERR_WORKSPACE",
                     "NSA_ERR_CUDA", "NSA_ERR_TIMEOUT"]
    assert nsa.nsa_status_string(99) == "NSA_ERR_UNKNOWN"


@pytest.mark.parametrize("lens,l,d", [([1024], 32, 16), ([16384], 32, 16), ([131072], 64, 32),
                                      ([65536] * 4, 128, 64), ([31, 0, 32, 33, 47, 48, 500], 32, 16),
                                      ([5, 100, 7], 48, 16)])
def test_compress_out_len_matches_oracle(lib, lens, l, d):
    cu = np.cumsum(lens).astype(np.int32)
    assert nsa.nsa_compress_out_len(cu, l, d).tolist() == oracle.compress_len(cu, l, d).tolist()


def test_compress_out_len_rejects_decreasing_prefix(lib):
    with pytest.raises(ValueError):
        nsa.nsa_compress_out_len([10, 5], 32, 16)


def _ws(**kw):
    a = dict(head_num=64, n2=4, d1=128, d2=128, l=32, d=16, lp=64, count=16,
             cu_seqlens_q=[16384], cu_cmp_kv=[1023], cu_sel_kv=[256])
    a.update(kw)
    return nsa.nsa_compress_attention_workspace_size(**a)


def test_workspace_size_is_positive_and_grows_with_tiles(lib):
    small = _ws(cu_seqlens_q=[1024], cu_cmp_kv=[63], cu_sel_kv=[16])
    big = _ws()
    assert 256 < small < big


@pytest.mark.parametrize("kw", [
    dict(l=24), dict(d=8), dict(lp=40), dict(l=144), dict(d=80), dict(lp=144),
    dict(l=16, d=32), dict(lp=16, l=32), dict(lp=48, d=32, l=32), dict(count=0), dict(count=33),
    dict(d1=64, d2=128), dict(d1=120), dict(d2=40), dict(head_num=6, n2=4), dict(head_num=2, n2=4),
    dict(cu_seqlens_q=[10, 5], cu_cmp_kv=[0, 0], cu_sel_kv=[1, 1]),
])
def test_attention_constraints_invalid(lib, kw):
    with pytest.raises(ValueError, match="INVALID_ARG"):
        _ws(**kw)


@pytest.mark.parametrize("kw", [
    dict(l=48, d=32, lp=96),            # l % d != 0: l/d is not an integer in step 4
    dict(d1=272, d2=128),               # head dim beyond 256
    dict(head_num=256, n2=1),           # 256 query heads per KV group
])
def test_attention_constraints_unsupported(lib, kw):
    with pytest.raises(ValueError, match="UNSUPPORTED"):
        _ws(**kw)


def _call_attention(lib, **kw):
    a = dict(q=4096, kcmp=4096, vcmp=4096, scale=0.1, head_num=64, l=32, d=16, lp=64, count=16,
             cq=[16384], cc=[1023], cs=[256], n2=4, d1=128, d2=128, dtype=0, out=4096, tk=4096,
             smax=4096, ssum=4096, ws=4096, wsb=1 << 30)
    a.update(kw)
    arr = lambda x: np.ascontiguousarray(np.asarray(x, np.int32))
    cq, cc, cs = arr(a["cq"]), arr(a["cc"]), arr(a["cs"])
    ip = lambda x: x.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return lib.nsa_compress_attention(a["q"], a["kcmp"], a["vcmp"], a["scale"], a["head_num"], a["l"],
                                      a["d"], a["lp"], a["count"], ip(cq), ip(cc), ip(cs), cq.size,
                                      a["n2"], a["d1"], a["d2"], a["dtype"], a["out"], a["tk"],
                                      a["smax"], a["ssum"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(tk=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(q=4100), nsa.NSA_ERR_INVALID_ARG),           # misaligned
    (dict(dtype=7), nsa.NSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), nsa.NSA_ERR_INVALID_ARG),
    (dict(ws=None), nsa.NSA_ERR_WORKSPACE),
    (dict(ws=4096 + 16), nsa.NSA_ERR_WORKSPACE),       # workspace must be 256-byte aligned
    (dict(wsb=64), nsa.NSA_ERR_WORKSPACE),             # undersized
    (dict(count=40), nsa.NSA_ERR_INVALID_ARG),
])
def test_attention_rejects_before_launch(lib, kw, status):
    assert _call_attention(lib, **kw) == status


def _call_compress(lib, **kw):
    a = dict(k=4096, v=4096, w=4096, l=32, d=16, cu=[1024], n2=4, d1=128, d2=128, dtype=0,
             kc=4096, vc=4096)
    a.update(kw)
    cu = np.ascontiguousarray(np.asarray(a["cu"], np.int32))
    return lib.nsa_compress(a["k"], a["v"], a["w"], a["l"], a["d"],
                            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size, a["n2"],
                            a["d1"], a["d2"], a["dtype"], a["kc"], a["vc"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(k=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(vc=None), nsa.NSA_ERR_INVALID_ARG),           # v given without vcmp
    (dict(l=24), nsa.NSA_ERR_INVALID_ARG),
    (dict(l=16, d=32), nsa.NSA_ERR_INVALID_ARG),        # l < d
    (dict(l=144), nsa.NSA_ERR_INVALID_ARG),
    (dict(d1=40), nsa.NSA_ERR_INVALID_ARG),
    (dict(d1=272), nsa.NSA_ERR_INVALID_ARG),
    (dict(k=4104), nsa.NSA_ERR_INVALID_ARG),            # misaligned
    (dict(cu=[10, 3]), nsa.NSA_ERR_INVALID_ARG),
    (dict(dtype=3), nsa.NSA_ERR_INVALID_ARG),
    (dict(n2=64, d1=256, d2=256), nsa.NSA_ERR_UNSUPPORTED),   # row wider than one CTA
])
def test_compress_rejects_before_launch(lib, kw, status):
    assert _call_compress(lib, **kw) == status


def test_python_binding_rejects_host_tensors(lib):
    import torch
    k = torch.zeros(64, 1, 16, dtype=torch.bfloat16)
    w = torch.zeros(32, 1, dtype=torch.bfloat16)
    with pytest.raises(TypeError, match="CUDA tensor"):
        nsa.nsa_compress(k, None, w, 32, 16, [64])


# ------------------------------------------------------------ selection attention
def _sws(**kw):
    a = dict(head_num=64, n2=4, d1=128, d2=128, lp=64, count=16, cu_seqlens_q=[16384], cu_seqlens_kv=[16384])
    a.update(kw)
    return nsa.nsa_select_attention_workspace_size(**a)


def test_select_workspace_size_is_positive_and_grows_with_tiles(lib):
    small = _sws(cu_seqlens_q=[1024], cu_seqlens_kv=[1024])
    big = _sws()
    assert 256 < small < big
    # short queries against long keys: the lists are sized by the keys' blocks
    assert _sws(cu_seqlens_q=[128], cu_seqlens_kv=[65536]) > _sws(cu_seqlens_q=[128], cu_seqlens_kv=[1024])


@pytest.mark.parametrize("kw", [
    dict(lp=40), dict(lp=8), dict(lp=144), dict(count=0), dict(count=33), dict(d1=120), dict(d2=40),
    dict(head_num=6, n2=4), dict(head_num=2, n2=4), dict(cu_seqlens_q=[10, 5], cu_seqlens_kv=[10, 20]),
    dict(cu_seqlens_q=[10, 20], cu_seqlens_kv=[10, 5]),
])
def test_select_constraints_invalid(lib, kw):
    with pytest.raises(ValueError, match="INVALID_ARG"):
        _sws(**kw)


@pytest.mark.parametrize("kw", [dict(d1=272), dict(d2=272), dict(head_num=256, n2=1)])
def test_select_constraints_unsupported(lib, kw):
    with pytest.raises(ValueError, match="UNSUPPORTED"):
        _sws(**kw)


def test_select_prefix_lists_must_pair_up(lib):
    with pytest.raises(ValueError):
        _sws(cu_seqlens_q=[100, 200], cu_seqlens_kv=[200])


def _call_select(lib, **kw):
    a = dict(q=4096, k=4096, v=4096, tk=4096, scale=0.1, head_num=64, lp=64, count=16, cq=[16384], ck=[16384],
             n2=4, d1=128, d2=128, dtype=0, out=4096, lse=4096, ws=4096, wsb=1 << 30)
    a.update(kw)
    arr = lambda x: np.ascontiguousarray(np.asarray(x, np.int32))
    cq, ck = arr(a["cq"]), arr(a["ck"])
    ip = lambda x: x.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return lib.nsa_select_attention(a["q"], a["k"], a["v"], a["tk"], a["scale"], a["head_num"], a["lp"],
                                    a["count"], ip(cq), ip(ck), cq.size, a["n2"], a["d1"], a["d2"], a["dtype"],
                                    a["out"], a["lse"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(tk=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(lse=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(k=4100), nsa.NSA_ERR_INVALID_ARG),            # misaligned
    (dict(tk=4098), nsa.NSA_ERR_INVALID_ARG),           # int32 list not 4-byte aligned
    (dict(lse=4097), nsa.NSA_ERR_INVALID_ARG),
    (dict(dtype=5), nsa.NSA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), nsa.NSA_ERR_INVALID_ARG),
    (dict(lp=24), nsa.NSA_ERR_INVALID_ARG),
    (dict(count=64), nsa.NSA_ERR_INVALID_ARG),
    (dict(ws=None), nsa.NSA_ERR_WORKSPACE),
    (dict(ws=4096 + 64), nsa.NSA_ERR_WORKSPACE),        # workspace must be 256-byte aligned
    (dict(wsb=256), nsa.NSA_ERR_WORKSPACE),             # undersized
    (dict(cq=[0], ck=[16384]), nsa.NSA_OK),             # no query rows: nothing to launch
])
def test_select_rejects_before_launch(lib, kw, status):
    assert _call_select(lib, **kw) == status


def _call_masked(lib, **kw):
    a = dict(q=4096, kcmp=4096, vcmp=4096, scale=0.1, head_num=64, l=32, d=16, lp=64, count=16,
             cq=[16384], cc=[1023], cs=[256], n2=4, d1=128, d2=128, dtype=0, am=4096, ar=16384, ac=1023,
             tm=4096, tr=16384, tc=256, out=4096, tk=4096, smax=4096, ssum=4096, ws=4096, wsb=1 << 30)
    a.update(kw)
    arr = lambda x: np.ascontiguousarray(np.asarray(x, np.int32))
    cq, cc, cs = arr(a["cq"]), arr(a["cc"]), arr(a["cs"])
    ip = lambda x: x.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return lib.nsa_compress_attention_masked(
        a["q"], a["kcmp"], a["vcmp"], a["scale"], a["head_num"], a["l"], a["d"], a["lp"], a["count"], ip(cq),
        ip(cc), ip(cs), cq.size, a["n2"], a["d1"], a["d2"], a["dtype"], a["am"], a["ar"], a["ac"], a["tm"],
        a["tr"], a["tc"], a["out"], a["tk"], a["smax"], a["ssum"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(ar=16383), nsa.NSA_ERR_INVALID_ARG),          # fewer mask rows than queries
    (dict(ac=1022), nsa.NSA_ERR_INVALID_ARG),           # fewer columns than compressed blocks
    (dict(tr=100), nsa.NSA_ERR_INVALID_ARG),
    (dict(tc=255), nsa.NSA_ERR_INVALID_ARG),            # fewer columns than selection blocks
    (dict(cq=[10, 5], cc=[0, 0], cs=[1, 1]), nsa.NSA_ERR_INVALID_ARG),
    (dict(q=None), nsa.NSA_ERR_INVALID_ARG),
    (dict(ws=None), nsa.NSA_ERR_WORKSPACE),
    (dict(am=None, ar=0, ac=0, ws=4096 + 8), nsa.NSA_ERR_WORKSPACE),   # a mask may be absent
])
def test_masked_attention_rejects_before_launch(lib, kw, status):
    assert _call_masked(lib, **kw) == status


def test_debug_library_exports_every_declared_symbol():
    # the NSA_DEBUG build (device bounds checks) offers the same C ABI
    path = _build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(dbg, name), name
