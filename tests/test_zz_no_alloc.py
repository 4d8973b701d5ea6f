"""The no-allocation variant of the compressed-attention entry point.

nsa_compress_attention_noalloc serves callers that cannot allocate device
memory (for instance an application that has reserved nearly all GPU memory
for its own pools, or a plugin handed only its tensors).  It takes inputs and
outputs only and runs in the library's fixed scratch array.  This file checks,
through the C ABI, that two calls in a row reproduce the regular entry point
within the parity tolerances with a clean device error word after each
(nsa_noalloc_status), and that oversized problems are refused.  It is
named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _inputs(wl):
    x = wl.generate(device="cuda")
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    kc = torch.from_numpy(kc).to(wl.torch_dtype).cuda()
    vc = torch.from_numpy(vc).to(wl.torch_dtype).cuda()
    return x, kc, vc, cuc


def _empty_outputs(wl, t1):
    return (torch.full((t1, wl.n1, wl.d2), float("nan"), dtype=wl.torch_dtype, device="cuda"),
            torch.full((t1, wl.n2, wl.count), -7, dtype=torch.int32, device="cuda"),
            torch.full((t1, wl.n1, 8), float("nan"), dtype=torch.float32, device="cuda"),
            torch.full((t1, wl.n1, 8), float("nan"), dtype=torch.float32, device="cuda"))


def _close(a, b):
    # same bars as the parity tests: output max-abs 1e-2, statistics 1e-3
    # relative (floor 1e-6), top-k index sets identical (same kernel, same inputs)
    assert torch.isfinite(a[0].float()).all()
    assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2
    for i in (2, 3):
        x, y = a[i].double(), b[i].double()
        same_inf = torch.isinf(x) == torch.isinf(y)
        assert same_inf.all()
        fin = ~torch.isinf(y)
        err = (x[fin] - y[fin]).abs()
        assert (err <= 1e-3 * y[fin].abs().clamp_min(1e-3) + 1e-6).all()
    assert torch.equal(a[1], b[1])


@pytest.mark.parametrize("wl", [workloads.TINY, workloads.SINGLE_16K], ids=lambda w: w.name)
def test_noalloc_matches_regular_entry_point_twice(nsa, wl):
    x, kc, vc, cuc = _inputs(wl)
    args = (x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
            x["cu_sel_kv"])
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    ref = nsa.nsa_compress_attention(*args, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    t1 = x["q"].shape[0]
    for _ in range(2):                       # the scratch keeps the previous call's contents
        got = nsa.nsa_compress_attention_noalloc(*args, out=_empty_outputs(wl, t1))
        # the error word lives in the fixed scratch array: read it through the
        # status call made for it (it also synchronises the stream)
        assert nsa.nsa_noalloc_status() == 0
        _close(got, ref)


def test_noalloc_refuses_problems_beyond_the_fixed_scratch(nsa):
    # l' = d = 16 over 300000 tokens: 18750 compressed blocks, each a
    # selection anchor, so one CTA's importance scratch (two slots of 128 rows
    # of ~19000 floats) alone exceeds 16 MiB; refused before anything is
    # enqueued
    S, n, dd = 300000, 1, 16
    cuc = nsa.nsa_compress_out_len([S], 16, 16)
    wl = workloads.Workload("big", (S,), n, n, dd, dd, 16, 16, 16, 8, 0.25)
    need = nsa.nsa_compress_attention_workspace_size(n, n, dd, dd, 16, 16, 16, 8, [S], cuc, [S // 16])
    assert need > (16 << 20)
    q = torch.zeros(S, n, dd, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(int(cuc[-1]), n, dd, dtype=torch.bfloat16, device="cuda")
    outs = _empty_outputs(wl, S)
    with pytest.raises(Exception, match="NSA_ERR_WORKSPACE"):
        nsa.nsa_compress_attention_noalloc(q, kv, kv, 0.25, n, 16, 16, 16, 8, [S], cuc, [S // 16], out=outs)
