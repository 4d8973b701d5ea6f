"""Parity of the fused CUDA compressed-attention kernel with the fp64 oracle.

Both sides get the same storage-dtype kcmp / vcmp (made by the oracle's
compression of seeded raw K/V), so the comparison isolates steps 1-7.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_attention, check_compress

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _prepare(wl, device="cpu"):
    x = wl.generate(device=device)
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    k, v, w = x["k"].cpu(), x["v"].cpu(), x["w"].cpu()
    kc, cuc = oracle.compress(k, w, wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(v, w, wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    tdt = wl.torch_dtype
    kc_t = torch.from_numpy(kc).to(tdt)
    vc_t = torch.from_numpy(vc).to(tdt)
    return x, kc_t, vc_t, cuc


def _run_both(nsa, wl, rows=None, device="cpu"):
    x, kc, vc, cuc = _prepare(wl, device)
    q = x["q"]
    qd = q if q.is_cuda else q.cuda()
    res = _attn(nsa, qd, kc.cuda(), vc.cuda(), wl, x, cuc)
    if rows is None:
        qo = q.cpu()
        ref = oracle.compress_attention(qo, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                        x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    else:
        rows = np.asarray(rows, dtype=np.int64)
        qs = q.index_select(0, torch.from_numpy(rows).to(q.device)).cpu()
        ref = oracle.compress_attention(qs, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                        x["cu_seqlens_q"], cuc, x["cu_sel_kv"], rows=rows,
                                        q_rows_only=True)
    return res, ref, x, (kc, vc, cuc)


def _attn(nsa, q, kc, vc, wl, x, cuc):
    """Runs the CUDA path and asserts that no device-side wait gave up."""
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
        x["cu_sel_kv"]), dtype=torch.uint8, device=q.device)
    res = nsa.nsa_compress_attention(q, kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                     x["cu_seqlens_q"], cuc, x["cu_sel_kv"], workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0, hex(int(ws[:4].view(torch.int32).item()))
    return res


def _wl(seqs, n1, n2, d1, d2, l, d, lp, count, dtype="bf16", seed=7, q_last=None, std=1.0):
    return workloads.Workload("case", tuple(seqs), n1, n2, d1, d2, l, d, lp, count, d1 ** -0.5,
                              dtype, seed=seed, std=std, q_last=q_last)


def test_tiny_workload_full(nsa):
    res, ref, _, _ = _run_both(nsa, workloads.TINY)
    rep = check_attention(res, ref, workloads.TINY.count)
    print(rep)


GROUPS = [(4, 1), (8, 8), (12, 4), (16, 2), (32, 2), (64, 2), (64, 1), (128, 1)]


@pytest.mark.parametrize("n1,n2", GROUPS, ids=lambda v: str(v))
def test_group_sizes(nsa, n1, n2):
    # several KV tiles (n_cmp = 155) with a ragged last tile and a ragged token tail
    wl = _wl([2500], n1, n2, 64, 64, 32, 16, 64, 8)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


BANDS = [(16, 16, 16), (32, 16, 32), (32, 16, 48), (32, 16, 64), (64, 16, 80), (32, 16, 96),
         (64, 16, 112), (128, 16, 128), (64, 32, 64), (128, 64, 128), (64, 32, 128), (48, 16, 96)]


@pytest.mark.parametrize("l,d,lp", BANDS, ids=lambda v: str(v))
def test_band_parameters(nsa, l, d, lp):
    wl = _wl([3000, 700], 16, 2, 64, 64, l, d, lp, 6)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


# D2 > 128 runs one M-tile per work item (two score buffers and O of up to 256
# columns in tensor memory); the others run two M-tiles per item
@pytest.mark.parametrize("d1,d2,dtype", [(64, 64, "fp16"), (128, 128, "bf16"), (192, 128, "fp16"),
                                         (96, 48, "bf16"), (128, 64, "bf16"), (32, 16, "fp16"),
                                         (256, 256, "bf16"), (160, 144, "fp16")])
def test_head_dims_and_dtypes(nsa, d1, d2, dtype):
    wl = _wl([1800, 333], 8, 2, d1, d2, 64, 32, 64, 16, dtype=dtype)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


def test_varlen_with_empty_and_short_sequences(nsa):
    wl = _wl([0, 900, 31, 47, 1, 2049, 16, 600], 16, 4, 64, 64, 32, 16, 64, 8)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


@pytest.mark.parametrize("count", [1, 32])
def test_count_extremes(nsa, count):
    wl = _wl([1500], 8, 1, 64, 64, 32, 16, 32, count)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


def test_short_queries_bottom_right_aligned(nsa):
    wl = _wl([4096, 3000, 2001], 32, 4, 64, 64, 64, 32, 64, 16, q_last=100)
    res, ref, _, _ = _run_both(nsa, wl)
    check_attention(res, ref, wl.count)


def test_score_buffer_in_global_memory(nsa):
    # one head per group (128 tokens per tile) and many selection blocks:
    # the per-token score buffers do not fit on chip and go to the workspace
    wl = _wl([20000], 2, 2, 64, 64, 16, 16, 16, 32)
    res, ref, _, _ = _run_both(nsa, wl, rows=workloads.sample_rows(np.array([20000], np.int32),
                                                                      first=300, last=300, every=37))
    check_attention(res, ref, wl.count)


def _direct(nsa, q, kc, vc, scale, l, d, lp, count, seqs, out_rel=0.0):
    """GPU vs oracle on given q / kcmp / vcmp (storage dtype, CPU tensors)."""
    cu = np.cumsum(seqs).astype(np.int32)
    cuc = oracle.compress_len(cu, l, d)
    cus = np.cumsum([-(-s_ // lp) for s_ in seqs]).astype(np.int32)
    n1, n2 = q.shape[1], kc.shape[1]
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(n1, n2, q.shape[2], vc.shape[2], l, d, lp, count,
                                                               cu, cuc, cus), dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention(q.cuda(), kc.cuda(), vc.cuda(), scale, n1, l, d, lp, count, cu, cuc, cus,
                                     workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0, hex(int(ws[:4].view(torch.int32).item()))
    ref = oracle.compress_attention(q, kc, vc, scale, l, d, lp, count, cu, cuc, cus)
    return check_attention(res, ref, count, out_rel=out_rel)


@pytest.mark.parametrize("step,dd", [(40, 64), (7, 64), (7, 256)], ids=["s40", "s7", "s7_d256"])
def test_reference_maximum_moves(nsa, step, dd):
    """Scores with a staircase offset: every `step` compressed blocks the
    largest score of a row jumps by 10 (natural units, about 14 in log2), more
    than the kernel lets P grow over its reference maximum, so the reference
    moves inside KV tiles (chunks after the first), across KV tiles (O and L
    rescaled) and, with step 7, several times per tile; D = 256 runs the
    one-pipeline form, whose O rescale waits for the previous P V."""
    g = torch.Generator().manual_seed(11)
    S, n1, n2, l, d, lp, count = 3000, 16, 2, 32, 16, 64, 8
    n_cmp = (S - l) // d + 1
    scale = dd ** -0.5
    q = torch.randn(S, n1, dd, generator=g)
    q[:, :, 0] = 1.0
    kc = torch.randn(n_cmp, n2, dd, generator=g)
    kc[:, :, 0] = (10.0 / scale) * torch.div(torch.arange(n_cmp), step, rounding_mode="floor")[:, None].float() \
        / max(1, (n_cmp // step) // 8)
    vc = torch.randn(n_cmp, n2, dd, generator=g)
    # rows end up on one or two value rows (|v| up to about 4.5): the bf16
    # rounding of the output itself exceeds 1e-2 there, hence the relative term
    rep = _direct(nsa, q.to(torch.bfloat16), kc.to(torch.bfloat16), vc.to(torch.bfloat16), scale, l, d, lp,
                  count, [S], out_rel=2.0 ** -7)
    print(rep)


def _staircase_short(nsa, n1, n2, dd, seqs, nq, step, l=32, d=16, lp=64, count=8):
    """The last nq queries of each sequence against keys whose first component
    climbs by 10/3 (natural units) every `step` blocks of a sequence."""
    g = torch.Generator().manual_seed(11)
    scale = dd ** -0.5
    cu = np.cumsum(seqs).astype(np.int32)
    cuc = oracle.compress_len(cu, l, d)
    cus = np.cumsum([-(-s_ // lp) for s_ in seqs]).astype(np.int32)
    cuq = np.cumsum([min(nq, s_) for s_ in seqs]).astype(np.int32)
    q = torch.randn(int(cuq[-1]), n1, dd, generator=g)
    q[:, :, 0] = 1.0
    kc = torch.randn(int(cuc[-1]), n2, dd, generator=g)
    pos = torch.cat([torch.arange(int(cuc[i]) - (int(cuc[i - 1]) if i else 0)) for i in range(len(seqs))])
    kc[:, :, 0] = (10.0 / scale) * torch.div(pos, step, rounding_mode="floor")[:, None].float() / 3.0
    vc = torch.randn(int(cuc[-1]), n2, dd, generator=g)
    q, kc, vc = q.to(torch.bfloat16), kc.to(torch.bfloat16), vc.to(torch.bfloat16)
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(n1, n2, dd, dd, l, d, lp, count, cuq, cuc, cus),
                     dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention(q.cuda(), kc.cuda(), vc.cuda(), scale, n1, l, d, lp, count, cuq, cuc, cus,
                                     workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    ref = oracle.compress_attention(q, kc, vc, scale, l, d, lp, count, cuq, cuc, cus)
    return check_attention(res, ref, count, out_rel=2.0 ** -7)


@pytest.mark.parametrize("n1,dd,nq,mixed", [(16, 256, 16, False), (16, 256, 16, True), (128, 256, 3000, False),
                                             (24, 256, 3000, True)],
                         ids=["g8_d256_16q", "g8_d256_16q_short_seqs", "g64_d256", "g12_d256"])
def test_one_pass_one_pipeline(nsa, n1, dd, nq, mixed):
    """The one-pass kernel with one pipeline and two score buffers (D2 > 128),
    many items per CTA and a reference maximum that moves: G = 8 with at most
    one M-tile of queries per sequence (300 sequences of 16 queries; or
    sequences as short as 16 tokens, whose rows attend to nothing or to one
    block), G = 64 (above the two-pass range) and G = 12 (not a power of two)
    over whole sequences, short ones among them."""
    if nq == 16:
        seqs = [16, 31, 32, 40, 47, 100, 300, 1000, 3000] * 30 if mixed else [3000 - 7 * (i % 50) for i in range(300)]
    else:
        seqs = [3000, 700, 40, 16] if mixed else [3000, 2500]
    print(_staircase_short(nsa, n1, 2, dd, seqs, nq, step=7))


@pytest.mark.parametrize("scale", [-0.125, 0.0])
def test_non_positive_scale(nsa, scale):
    g = torch.Generator().manual_seed(12)
    S, n1, n2, dd, l, d, lp, count = 1500, 8, 2, 64, 32, 16, 64, 8
    n_cmp = (S - l) // d + 1
    q = torch.randn(S, n1, dd, generator=g).to(torch.bfloat16)
    kc = (torch.randn(n_cmp, n2, dd, generator=g) * 0.3).to(torch.bfloat16)
    vc = torch.randn(n_cmp, n2, dd, generator=g).to(torch.bfloat16)
    _direct(nsa, q, kc, vc, scale, l, d, lp, count, [S])


def test_deterministic_and_status(nsa):
    wl = _wl([3000], 32, 2, 128, 128, 32, 16, 64, 16)
    x, kc, vc, cuc = _prepare(wl)
    args = (x["q"].cuda(), kc.cuda(), vc.cuda(), wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
            x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
        x["cu_sel_kv"]), dtype=torch.uint8, device="cuda")
    a = nsa.nsa_compress_attention(*args, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    b = nsa.nsa_compress_attention(*args, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1], b[1])
    assert torch.equal(a[2], b[2]) and torch.equal(a[3], b[3])


def test_end_to_end_gpu_compress_then_attention(nsa):
    """GPU compress feeding GPU attention, checked in two stages: the GPU's
    kcmp / vcmp against the oracle's compression (1 ulp rule), then the GPU
    attention against the oracle's attention run on those same GPU-made
    kcmp / vcmp, with the full tie-aware top-k rule."""
    wl = _wl([4000, 1234], 32, 4, 128, 128, 32, 16, 64, 16)
    x = wl.generate()
    kc, vc = nsa.nsa_compress(x["k"].cuda(), x["v"].cuda(), x["w"].cuda(), wl.l, wl.d, x["cu_seqlens"])
    assert nsa.nsa_compress_status() == 0
    check_compress(kc, x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], oracle.BF16)
    check_compress(vc, x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], oracle.BF16)
    cuc = nsa.nsa_compress_out_len(x["cu_seqlens"], wl.l, wl.d)
    res = _attn(nsa, x["q"].cuda(), kc, vc, wl, x, cuc)
    ref = oracle.compress_attention(x["q"], kc.cpu(), vc.cpu(), wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                    x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    rep = check_attention(res, ref, wl.count)
    print("end-to-end", rep)


# ---------------------------------------------------------------- full size
def _sample(wl, x, first, last, every):
    return workloads.sample_rows(x["cu_seqlens_q"], first=first, last=last, every=every)


@pytest.mark.parametrize("wl,sample", [
    (workloads.SINGLE_16K, (256, 512, 61)),
    (workloads.VARLEN_8, (96, 128, 211)),
    (workloads.LONG_128K, (64, 160, 1999)),
    (workloads.SHORTQ_4x64K, None),
], ids=lambda v: getattr(v, "name", "s"))
def test_full_size_workloads(nsa, wl, sample):
    """The benchmark's launch configuration at full size; sampled rows are
    checked one by one against the oracle (all rows for the short-query case)."""
    x, kc, vc, cuc = _prepare(wl, device="cuda")
    rows = None if sample is None else workloads.sample_rows(x["cu_seqlens_q"], *sample)
    q = x["q"]
    res = _attn(nsa, q, kc.cuda(), vc.cuda(), wl, x, cuc)
    if rows is None:
        qo = q.cpu()
        ref = oracle.compress_attention(qo, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                        x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    else:
        qs = q.index_select(0, torch.from_numpy(rows).cuda()).cpu()
        ref = oracle.compress_attention(qs, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                        x["cu_seqlens_q"], cuc, x["cu_sel_kv"], rows=rows,
                                        q_rows_only=True)
    rep = check_attention(res, ref, wl.count)
    print(wl.name, rep)
