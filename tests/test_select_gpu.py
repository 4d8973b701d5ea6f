"""Parity of the CUDA selection attention (nsa_select_attention) with the fp64
oracle: attention over the raw K/V blocks of l' tokens listed per (query row,
KV group), as the compressed branch's top-k lists them.  Both sides get the
same storage-dtype q, k, v and the same index lists."""
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


def _lists(cq, ck, n2, count, lp, seed, holes=True):
    """Random index lists: per (row, group) up to `count` distinct blocks of the
    row's sequence that start at or before the row's key position, ascending,
    then -1 padding."""
    rng = np.random.default_rng(seed)
    T1 = int(cq[-1])
    sel = np.full((T1, n2, count), -1, np.int32)
    q0, k0 = 0, 0
    for b in range(len(cq)):
        Sq, Skv = int(cq[b]) - q0, int(ck[b]) - k0
        for tl in range(Sq):
            t = tl + Skv - Sq
            if t < 0:
                continue
            nb = t // lp + 1
            for g in range(n2):
                m = int(rng.integers(1 if not holes else 0, min(count, nb) + 1))
                pick = np.sort(rng.choice(nb, size=m, replace=False)).astype(np.int32)
                sel[q0 + tl, g, :m] = pick
        q0, k0 = int(cq[b]), int(ck[b])
    return sel


def _run(nsa, seqs_q, seqs_kv, n1, n2, d1, d2, lp, count, dtype="bf16", seed=0, sel=None, rows=None):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    g = torch.Generator().manual_seed(seed)
    cq = np.cumsum(seqs_q).astype(np.int32)
    ck = np.cumsum(seqs_kv).astype(np.int32)
    T1, T2 = int(cq[-1]), int(ck[-1])
    q = torch.randn(T1, n1, d1, generator=g).to(tdt)
    k = torch.randn(T2, n2, d1, generator=g).to(tdt)
    v = torch.randn(T2, n2, d2, generator=g).to(tdt)
    if sel is None:
        sel = _lists(cq, ck, n2, count, lp, seed)
    scale = d1 ** -0.5
    out, lse = nsa.nsa_select_attention(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(sel).cuda(), scale, n1,
                                        lp, cq, ck)
    torch.cuda.synchronize()
    if rows is None:
        ref = oracle.select_attention(q.float(), k.float(), v.float(), sel, scale, lp, count, cq, ck)
        rows = np.arange(T1)
    else:
        ref = oracle.select_attention(q.float()[rows], k.float(), v.float(), sel, scale, lp, count, cq, ck,
                                      rows=rows, q_rows_only=True)
    return out.float().cpu().numpy()[rows], lse.cpu().numpy()[rows], ref


def _check(out, lse, ref, out_tol=1e-2, lse_tol=1e-3):
    """attention_out within 1e-2 + 2^-7 |ref| element-wise: the output is rounded
    to the storage dtype once (half an ulp: 2^-8 |ref| for bf16) after P was
    (another 2^-8 relative per term); rows that attend to few keys keep
    magnitudes of a single value row, where an absolute 1e-2 alone is below one
    bf16 ulp.  softmax_lse within 1e-3 absolute (fp32 sums of 2^x terms)."""
    empty = np.isneginf(ref["lse"])
    assert (np.isneginf(lse) == empty).all(), "empty rows must be exactly -inf"
    assert (out[empty] == 0).all()
    assert np.isfinite(out).all()
    if out.size:
        excess = np.abs(out - ref["out"]) - (out_tol + 2.0 ** -7 * np.abs(ref["out"]))
        assert excess.max() <= 0, f"attention_out off by {excess.max()} beyond the bound"
    if (~empty).any():
        lerr = np.abs(lse[~empty] - ref["lse"][~empty]).max()
        assert lerr <= lse_tol, f"softmax_lse max abs err {lerr}"


def test_small_case(nsa):
    out, lse, ref = _run(nsa, [1000], [1000], 4, 1, 64, 64, 64, 8)
    _check(out, lse, ref)


@pytest.mark.parametrize("n1,n2", [(4, 4), (8, 1), (32, 2), (16, 1), (64, 2), (128, 1), (6, 2)],
                         ids=lambda v: str(v))
def test_group_sizes(nsa, n1, n2):
    out, lse, ref = _run(nsa, [700, 333], [700, 333], n1, n2, 64, 64, 32, 6, seed=1)
    _check(out, lse, ref)


@pytest.mark.parametrize("lp", [16, 32, 48, 64, 80, 96, 112, 128])
def test_block_sizes(nsa, lp):
    out, lse, ref = _run(nsa, [1500], [1500], 16, 2, 64, 64, lp, 5, seed=2)
    _check(out, lse, ref)


@pytest.mark.parametrize("d1,d2,dtype", [(128, 128, "bf16"), (192, 128, "fp16"), (64, 256, "bf16")])
def test_head_dims_and_dtypes(nsa, d1, d2, dtype):
    out, lse, ref = _run(nsa, [900], [900], 8, 2, d1, d2, 64, 8, dtype=dtype, seed=3)
    _check(out, lse, ref)


def test_short_queries_varlen_and_empty(nsa):
    # bottom-right aligned short queries, an empty query sequence, a sequence
    # shorter than one block, and lists with repeats and out-of-range entries
    seqs_q, seqs_kv = [40, 0, 7, 300], [900, 50, 7, 300]
    cq, ck = np.cumsum(seqs_q).astype(np.int32), np.cumsum(seqs_kv).astype(np.int32)
    sel = _lists(cq, ck, 2, 6, 32, seed=4)
    sel[::5, :, 1] = sel[::5, :, 0]          # a repeat
    sel[::7, :, 2] = 10 ** 6                 # past the sequence
    out, lse, ref = _run(nsa, seqs_q, seqs_kv, 8, 2, 64, 64, 32, 6, seed=4, sel=sel)
    _check(out, lse, ref)


def test_count_extremes(nsa):
    for count in (1, 32):
        out, lse, ref = _run(nsa, [2000], [2000], 16, 4, 64, 64, 16, count, seed=5)
        _check(out, lse, ref)


@pytest.mark.parametrize("name,first,last,every", [
    ("single_s16384_n64_n4_d128", 64, 64, 257),
    ("varlen8_t158963_n32_n2_d192x128_fp16", 32, 32, 997),
    ("long_s131072_n128_n8_d128", 48, 48, 2039),
    ("compress_t262144_shortq_4x128_n64_n8_d128", 128, 128, 1),
], ids=["16k", "varlen", "long", "shortq"])
def test_pipeline_on_full_workloads(nsa, name, first, last, every):
    """Compress -> compressed attention -> selection attention on a workload at
    full size (the 16K one is the bench's; varlen runs fp16 with D1=192, the long
    one l'=128 and 32-entry lists, the short-query one bottom-right aligned
    queries).  Sampled rows against the oracle fed with the GPU's own top-k
    lists; every row of the short-query case."""
    wl = workloads.WORKLOADS[name]
    x = wl.generate(device="cuda")
    cuc = nsa.nsa_compress_out_len(x["cu_seqlens"], wl.l, wl.d)
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"])
    _, tk, _, _ = nsa.nsa_compress_attention(x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                             x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    out, lse = nsa.nsa_select_attention(x["q"], x["k"], x["v"], tk, wl.scale, wl.n1, wl.lp,
                                        x["cu_seqlens_q"], x["cu_seqlens"])
    torch.cuda.synchronize()
    rows = workloads.sample_rows(x["cu_seqlens_q"], first=first, last=last, every=every)
    sel = tk.cpu().numpy()
    rows_t = torch.from_numpy(rows).cuda()
    ref = oracle.select_attention(x["q"].index_select(0, rows_t).float().cpu(), x["k"].float().cpu(),
                                  x["v"].float().cpu(), sel, wl.scale, wl.lp, wl.count, x["cu_seqlens_q"],
                                  x["cu_seqlens"], rows=rows, q_rows_only=True)
    _check(out.index_select(0, rows_t).float().cpu().numpy(), lse.index_select(0, rows_t).cpu().numpy(), ref)


def test_deterministic_and_status(nsa):
    seqs = [1200]
    cq = np.cumsum(seqs).astype(np.int32)
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1200, 16, 64, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1200, 2, 64, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1200, 2, 64, generator=g).to(torch.bfloat16).cuda()
    sel = torch.from_numpy(_lists(cq, cq, 2, 8, 64, seed=9)).cuda()
    ws = torch.empty(nsa.nsa_select_attention_workspace_size(16, 2, 64, 64, 64, 8, cq, cq), dtype=torch.uint8,
                     device="cuda")
    a = nsa.nsa_select_attention(q, k, v, sel, 0.125, 16, 64, cq, cq, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    b = nsa.nsa_select_attention(q, k, v, sel, 0.125, 16, 64, cq, cq, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)) and torch.equal(a[1], b[1])
