"""Parity of the backward kernels with the fp64 oracle.

Compressed attention: both sides get the same storage-dtype q, kcmp, vcmp
(kcmp / vcmp from the oracle's compression of seeded raw K / V) and the same
seeded dout.  The GPU backward takes the GPU forward's attention_out and
statistics, as a training step does; the oracle differentiates its own exact
forward.  Compression: the same fp32 dkcmp / dvcmp on both sides.
Tolerances in parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_compress_dx, check_dw, check_grad

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _wl(seqs, n1, n2, d1, d2, l=32, d=16, lp=64, count=8, dtype="bf16", seed=11, q_last=None, std=1.0):
    return workloads.Workload("case", tuple(seqs), n1, n2, d1, d2, l, d, lp, count, d1 ** -0.5, dtype,
                              seed=seed, q_last=q_last, std=std)


def _inputs(wl):
    x = wl.generate()
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    kc = torch.from_numpy(kc).to(wl.torch_dtype)
    vc = torch.from_numpy(vc).to(wl.torch_dtype)
    return x, kc, vc, cuc, workloads.grad_output(wl)


def _gpu_backward(nsa, wl, x, kc, vc, cuc, dout):
    q, kcd, vcd = x["q"].cuda(), kc.cuda(), vc.cuda()
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    out, _, smax, ssum = nsa.nsa_compress_attention(q, kcd, vcd, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                                    x["cu_seqlens_q"], cuc, x["cu_sel_kv"], workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    wsb = torch.empty(nsa.nsa_compress_attention_backward_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, x["cu_seqlens_q"], cuc), dtype=torch.uint8, device="cuda")
    grads = nsa.nsa_compress_attention_backward(q, kcd, vcd, out, dout.cuda(), smax, ssum, wl.scale, wl.n1, wl.l,
                                                wl.d, x["cu_seqlens_q"], cuc, workspace=wsb)
    status = nsa.nsa_workspace_status(wsb)
    assert status == 0, hex(int(wsb[:4].view(torch.int32).item()))
    return [g.cpu() for g in grads]


def _check(nsa, wl, groups=None):
    x, kc, vc, cuc, dout = _inputs(wl)
    dq, dk, dv = _gpu_backward(nsa, wl, x, kc, vc, cuc, dout)
    G = wl.n1 // wl.n2
    reps = []
    for g in (range(wl.n2) if groups is None else groups):
        # one KV group's gradients depend only on its own heads
        hs = slice(g * G, (g + 1) * G)
        ref = oracle.compress_attention_backward(x["q"][:, hs], kc[:, g:g + 1], vc[:, g:g + 1], dout[:, hs],
                                                 wl.scale, wl.l, wl.d, x["cu_seqlens_q"], cuc)
        reps.append(check_grad(dq[:, hs], ref["dq"], f"dq[g{g}]"))
        reps.append(check_grad(dk[:, g:g + 1], ref["dkcmp"], f"dkcmp[g{g}]"))
        reps.append(check_grad(dv[:, g:g + 1], ref["dvcmp"], f"dvcmp[g{g}]"))
    return reps


def test_tiny_workload(nsa):
    print(_check(nsa, workloads.TINY))


def test_16k_workload_groups_0_and_3(nsa):
    # the 16K workload at full size; two of its four KV groups against the oracle
    print(_check(nsa, workloads.SINGLE_16K, groups=(0, 3)))


@pytest.mark.parametrize("n1,n2", [(4, 1), (12, 4), (16, 2), (128, 1), (8, 8)], ids=lambda v: str(v))
def test_group_sizes(nsa, n1, n2):
    # G = 3 leaves rows of the 128-row tile empty; G = 128 gives one token per tile
    _check(nsa, _wl([1200], n1, n2, 64, 64))


@pytest.mark.parametrize("d1,d2,dtype", [(128, 128, "bf16"), (192, 128, "fp16"), (256, 128, "bf16"),
                                          (192, 160, "bf16"), (128, 64, "fp16"), (16, 16, "bf16")],
                         ids=lambda v: str(v))
def test_head_dims(nsa, d1, d2, dtype):
    # D2 > 128 takes the two-pass dK / dV path
    _check(nsa, _wl([900], 8, 2, d1, d2, dtype=dtype))


@pytest.mark.parametrize("l,d", [(32, 16), (64, 32), (128, 64), (16, 16), (48, 16)], ids=lambda v: str(v))
def test_block_geometry(nsa, l, d):
    _check(nsa, _wl([1500], 8, 2, 64, 64, l=l, d=d, lp=max(l, 64)))


def test_varlen_empty_and_short_sequences(nsa):
    # an empty sequence, sequences shorter than one block, ragged tails
    _check(nsa, _wl([300, 0, 20, 777, 31, 2100], 16, 4, 64, 64))


def test_short_queries(nsa):
    # the last 70 queries of each sequence (query offset applied)
    _check(nsa, _wl([2000, 1500, 64], 16, 2, 64, 64, q_last=70))


def test_long_run_splits(nsa):
    # KV tiles whose query runs split into several partial slots
    _check(nsa, _wl([6000], 16, 1, 64, 64, std=0.5))


def test_deterministic(nsa):
    wl = _wl([3000], 16, 2, 64, 64)
    x, kc, vc, cuc, dout = _inputs(wl)
    a = _gpu_backward(nsa, wl, x, kc, vc, cuc, dout)
    b = _gpu_backward(nsa, wl, x, kc, vc, cuc, dout)
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int32), v.view(torch.int32))


def test_compress_backward(nsa):
    # ceil(l/d) = 2 windows per row (TINY, 64/32, 128/64), 1 (32/32), 4 (64/16), 8 (128/16) and
    # l % d != 0 (48/32)
    for wl in (workloads.TINY, _wl([300, 0, 20, 777], 8, 4, 64, 32, l=64, d=32, dtype="fp16"),
               _wl([1000], 8, 2, 128, 128, l=128, d=64), _wl([700, 33], 8, 2, 64, 64, l=32, d=32),
               _wl([900], 8, 2, 64, 64, l=64, d=16), _wl([1100, 200], 4, 2, 64, 32, l=128, d=16, lp=128),
               _wl([650], 8, 2, 64, 64, l=48, d=32, lp=64)):
        x = wl.generate()
        tc = int(nsa.nsa_compress_out_len(x["cu_seqlens"], wl.l, wl.d)[-1])
        g = torch.Generator().manual_seed(wl.seed + 2000)
        gk = torch.randn(tc, wl.n2, wl.d1, generator=g)
        gv = torch.randn(tc, wl.n2, wl.d2, generator=g)
        dk, dv, dw = nsa.nsa_compress_backward(x["k"].cuda(), x["v"].cuda(), x["w"].cuda(), gk.cuda(), gv.cuda(),
                                               wl.l, wl.d, x["cu_seqlens"])
        pk = check_compress_dx(dk, x["k"], x["w"], gk, wl.l, wl.d, x["cu_seqlens"])
        pv = check_compress_dx(dv, x["v"], x["w"], gv, wl.l, wl.d, x["cu_seqlens"])
        check_dw(dw, [pk, pv])
        # K alone
        dk1, dv1, dw1 = nsa.nsa_compress_backward(x["k"].cuda(), None, x["w"].cuda(), gk.cuda(), None, wl.l, wl.d,
                                                  x["cu_seqlens"])
        assert dv1 is None and torch.equal(dk1.cpu(), dk.cpu())
        check_dw(dw1, [pk])


def test_backward_refuses_bad_arguments(nsa):
    wl = _wl([500], 8, 2, 64, 64)
    x, kc, vc, cuc, dout = _inputs(wl)
    q = x["q"].cuda()
    out = torch.zeros(q.shape[0], 8, 64, dtype=q.dtype, device="cuda")
    st = torch.zeros(q.shape[0], 8, 8, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):   # D1 + D2 beyond what the kernels hold on chip
        big = torch.zeros(q.shape[0], 8, 256, dtype=q.dtype, device="cuda")
        kb = torch.zeros(kc.shape[0], 2, 256, dtype=q.dtype, device="cuda")
        nsa.nsa_compress_attention_backward(big, kb, kb, big, big, st, st, 0.1, 8, 32, 16, x["cu_seqlens_q"], cuc)
    with pytest.raises(ValueError):   # small workspace refused
        nsa.nsa_compress_attention_backward(q, kc.cuda(), vc.cuda(), out, out, st, st, 0.1, 8, 32, 16,
                                            x["cu_seqlens_q"], cuc,
                                            workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
