"""Parity of the CUDA compress kernel (nsa_compress) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_compress

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _case(lens, n2, d1, d2, l, d, dtype=torch.bfloat16, seed=0, std=1.0):
    g = torch.Generator().manual_seed(seed)
    T = int(sum(lens))
    k = (torch.randn(T, n2, d1, generator=g) * std).to(dtype)
    v = (torch.randn(T, n2, d2, generator=g) * std).to(dtype)
    w = (torch.rand(l, n2, generator=g) * (2.0 / l)).to(dtype)
    return k, v, w, np.cumsum(lens).astype(np.int32)


CASES = [
    # lens, n2, d1, d2, l, d
    ([1024], 1, 64, 64, 32, 16),
    ([777, 0, 31, 32, 33, 1500], 2, 64, 64, 32, 16),     # empty, S < l, S == l, ragged
    ([2000], 4, 128, 128, 64, 32),
    ([3001, 129], 8, 128, 128, 128, 64),
    ([900], 2, 192, 128, 64, 32),
    ([640, 50], 3, 48, 16, 48, 16),                    # l % d == 0, odd head dim
    ([1000], 2, 64, 32, 48, 32),                       # l % d != 0 (allowed for compress)
    ([513], 4, 256, 256, 128, 16),                     # b = 8 windows per row
    ([400], 1, 16, 16, 16, 16),                        # non-overlapping windows
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", CASES)
def test_compress_parity(nsa, case, dtype):
    lens, n2, d1, d2, l, d = case
    k, v, w, cu = _case(lens, n2, d1, d2, l, d, dtype)
    kc, vc = nsa.nsa_compress(k.cuda(), v.cuda(), w.cuda(), l, d, cu)
    torch.cuda.synchronize()
    assert nsa.nsa_compress_status() == 0
    dt = oracle.BF16 if dtype == torch.bfloat16 else oracle.FP16
    check_compress(kc, k, w, l, d, cu, dt)
    check_compress(vc, v, w, l, d, cu, dt)


def test_compress_k_only(nsa):
    k, v, w, cu = _case([700, 300], 2, 64, 64, 32, 16)
    kc, vc = nsa.nsa_compress(k.cuda(), None, w.cuda(), 32, 16, cu)
    assert nsa.nsa_compress_status() == 0
    assert vc is None
    check_compress(kc, k, w, 32, 16, cu, oracle.BF16)


def test_compress_one_hot_weight_is_exact_copy(nsa):
    k, v, w, cu = _case([1000, 77], 2, 128, 64, 64, 32)
    w = torch.zeros_like(w)
    w[5, 0] = 1.0
    w[63, 1] = 1.0
    kc, vc = nsa.nsa_compress(k.cuda(), v.cuda(), w.cuda(), 64, 32, cu)
    ref, _ = oracle.compress(k, w, 64, 32, cu, dtype=oracle.BF16)
    assert np.array_equal(kc.double().cpu().numpy(), ref)


def test_compress_deterministic(nsa):
    k, v, w, cu = _case([5000, 3000], 4, 128, 128, 32, 16, seed=3)
    k, v, w = k.cuda(), v.cuda(), w.cuda()
    a = nsa.nsa_compress(k, v, w, 32, 16, cu)
    b = nsa.nsa_compress(k, v, w, 32, 16, cu)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))


@pytest.mark.parametrize("wl", [workloads.SHORTQ_4x64K, workloads.SINGLE_16K, workloads.VARLEN_8],
                         ids=lambda w: w.name)
def test_compress_full_size_workloads(nsa, wl):
    """The compress launch of the benchmark at full size, every output checked."""
    x = wl.generate(device="cuda")
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"])
    assert nsa.nsa_compress_status() == 0
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    k, v, w = x["k"].cpu(), x["v"].cpu(), x["w"].cpu()
    check_compress(kc, k, w, wl.l, wl.d, x["cu_seqlens"], dt)
    check_compress(vc, v, w, wl.l, wl.d, x["cu_seqlens"], dt)
