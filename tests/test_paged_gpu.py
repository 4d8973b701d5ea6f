"""Paged compressed K/V (nsa_compress_attention_paged).

The paged call reads each compressed block through the block table; with the
same rows in the pages it must reproduce the contiguous call bit for bit.  The
decode shape (one query per sequence) is also checked against the fp64 oracle
on the contiguous tensors.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nsa():
    from sparse_long_context_nsa_b200 import _build
    _build.build()
    import sparse_long_context_nsa_b200 as m
    return m


def _wl(seqs, n1, n2, dd, l, d, lp, count, seed=31, q_last=None, dtype="bf16"):
    return workloads.Workload("case", tuple(seqs), n1, n2, dd, dd, l, d, lp, count, dd ** -0.5, dtype, seed=seed,
                              q_last=q_last)


def _inputs(wl):
    x = wl.generate()
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    return x, torch.from_numpy(kc).to(wl.torch_dtype), torch.from_numpy(vc).to(wl.torch_dtype), cuc


def _paginate(kc, vc, cuc, page_size, seed, spare=3, pad_entries=2, pad_value=-1):
    """Scatters every sequence's compressed rows into shuffled pages of a pool
    (unused pages and rows zero) and returns (kpool, vpool, block_table)."""
    ncs = np.diff(np.concatenate([[0], cuc]))
    npg = [-(-int(n) // page_size) for n in ncs]
    total = sum(npg) + spare
    rng = np.random.default_rng(seed)
    order = rng.permutation(total)
    n2, d1, d2 = kc.shape[1], kc.shape[2], vc.shape[2]
    kpool = torch.zeros(total, page_size, n2, d1, dtype=kc.dtype)
    vpool = torch.zeros(total, page_size, n2, d2, dtype=vc.dtype)
    width = max(1, max(npg)) + pad_entries
    table = np.full((len(ncs), width), pad_value, dtype=np.int32)
    nxt, start = 0, 0
    for b, n in enumerate(ncs):
        for j in range(npg[b]):
            pg = int(order[nxt])
            nxt += 1
            table[b, j] = pg
            rows = slice(start + j * page_size, start + min(n, (j + 1) * page_size))
            cnt = rows.stop - rows.start
            kpool[pg, :cnt] = kc[rows]
            vpool[pg, :cnt] = vc[rows]
        start += int(n)
    return kpool, vpool, torch.from_numpy(table)


def _both(nsa, wl, x, kc, vc, cuc, page_size, seed=0, pad_value=-1):
    q = x["q"].cuda()
    contiguous = nsa.nsa_compress_attention(q, kc.cuda(), vc.cuda(), wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                            x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    kp, vp, bt = _paginate(kc, vc, cuc, page_size, seed, pad_value=pad_value)
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    paged = nsa.nsa_compress_attention_paged(q, kp.cuda(), vp.cuda(), bt.cuda(), wl.scale, wl.n1, wl.l, wl.d, wl.lp,
                                             wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"], workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    return contiguous, paged


def _bitwise(a, b):
    for u, v in zip(a, b):
        u, v = u.cpu(), v.cpu()
        if u.dtype in (torch.bfloat16, torch.float16):
            u, v = u.view(torch.int16), v.view(torch.int16)
        elif u.dtype == torch.float32:
            u, v = u.view(torch.int32), v.view(torch.int32)
        assert torch.equal(u, v)


@pytest.mark.parametrize("page_size", [8, 16, 32, 64, 128])
def test_paged_equals_contiguous(nsa, page_size):
    # varlen with an empty sequence, sequences shorter than a block and ragged last pages
    wl = _wl([300, 0, 40, 777, 2100], 16, 4, 64, 32, 16, 64, 8)
    x, kc, vc, cuc = _inputs(wl)
    c, p = _both(nsa, wl, x, kc, vc, cuc, page_size, seed=page_size)
    _bitwise(c, p)


@pytest.mark.parametrize("page_size", [16, 32, 48, 96])
def test_paged_equals_contiguous_96_block_tiles(nsa, page_size):
    # l'/d = 3: KV tiles of 96 blocks, pages of a divisor of 96
    wl = _wl([1500, 333], 8, 2, 64, 32, 16, 48, 6, seed=32)
    x, kc, vc, cuc = _inputs(wl)
    c, p = _both(nsa, wl, x, kc, vc, cuc, page_size, seed=page_size, pad_value=1 << 30)
    _bitwise(c, p)


def test_decode_one_query_per_sequence(nsa):
    # one query per sequence: the last raw token of each, against every block
    lens = [int(n) for n in np.random.default_rng(33).integers(100, 5000, 12)]
    wl = _wl(lens, 16, 2, 128, 64, 32, 128, 16, seed=34, q_last=1)
    x, kc, vc, cuc = _inputs(wl)
    assert list(x["cu_seqlens_q"]) == list(range(1, 13))
    kp, vp, bt = _paginate(kc, vc, cuc, 64, seed=35)
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention_paged(x["q"].cuda(), kp.cuda(), vp.cuda(), bt.cuda(), wl.scale, wl.n1, wl.l,
                                           wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"],
                                           workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"])
    check_attention(res, ref, wl.count)


def test_decode_fp16_gqa_shapes(nsa):
    lens = [4096, 130, 4000, 2500]
    wl = _wl(lens, 64, 8, 128, 128, 64, 128, 32, seed=36, q_last=1, dtype="fp16")
    x, kc, vc, cuc = _inputs(wl)
    kp, vp, bt = _paginate(kc, vc, cuc, 128, seed=37)
    res = nsa.nsa_compress_attention_paged(x["q"].cuda(), kp.cuda(), vp.cuda(), bt.cuda(), wl.scale, wl.n1, wl.l,
                                           wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"])
    check_attention(res, ref, wl.count)


def test_paged_refuses_bad_arguments(nsa):
    wl = _wl([900], 8, 2, 64, 32, 16, 64, 5, seed=38)
    x, kc, vc, cuc = _inputs(wl)
    kp, vp, bt = _paginate(kc, vc, cuc, 32, seed=39, pad_entries=0)
    q = x["q"].cuda()
    wide = torch.zeros(1, 64, dtype=torch.int32, device="cuda")   # long enough for any page size here
    for bad_size in (20, 256):   # not a multiple of 8; does not divide the 128-block KV tile
        kb = torch.zeros(4, bad_size, *kp.shape[2:], dtype=kp.dtype, device="cuda")
        with pytest.raises(ValueError):
            nsa.nsa_compress_attention_paged(q, kb, kb, wide, wl.scale, wl.n1, wl.l, wl.d, wl.lp,
                                             wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    with pytest.raises(ValueError):   # a block-table row too short for the sequence's pages
        nsa.nsa_compress_attention_paged(q, kp.cuda(), vp.cuda(), bt[:, :-1].contiguous().cuda(), wl.scale,
                                         wl.n1, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])


def test_decode_workload_full_size_sampled_sequences(nsa):
    # the bench's decode step at full size; 8 of its 64 sequences against the oracle
    dw = workloads.DECODE_64x64K
    x = dw.generate(device="cuda")
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        dw.n1, dw.n2, dw.d1, dw.d2, dw.l, dw.d, dw.lp, dw.count, x["cu_seqlens_q"], x["cu_cmp_kv"], x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention_paged(x["q"], x["kcmp_pages"], x["vcmp_pages"], x["block_table"], dw.scale,
                                           dw.n1, dw.l, dw.d, dw.lp, dw.count, x["cu_seqlens_q"], x["cu_cmp_kv"],
                                           x["cu_sel_kv"], workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0, hex(int(ws[:4].view(torch.int32).item()))
    picks = [0, 9, 17, 31, 40, 52, 60, 63]
    bt = x["block_table"].cpu().numpy()
    kp, vp = x["kcmp_pages"].cpu(), x["vcmp_pages"].cpu()
    kc = torch.cat([kp[bt[b]].reshape(-1, dw.n2, dw.d1)[:dw.n_cmp] for b in picks])
    vc = torch.cat([vp[bt[b]].reshape(-1, dw.n2, dw.d2)[:dw.n_cmp] for b in picks])
    n = len(picks)
    ref = oracle.compress_attention(x["q"][picks].cpu(), kc, vc, dw.scale, dw.l, dw.d, dw.lp, dw.count,
                                    np.arange(1, n + 1, dtype=np.int32),
                                    (np.arange(1, n + 1) * dw.n_cmp).astype(np.int32),
                                    x["cu_sel_kv"][:n])
    sub = [t[picks] for t in res]
    check_attention(sub, ref, dw.count)


def _gather(pool, table, n_cmp_list):
    out = []
    for b, n in enumerate(n_cmp_list):
        out.append(pool[table[b].long()].reshape(-1, *pool.shape[2:])[:n])
    return torch.cat(out)


@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_compress_equals_contiguous(nsa, page_size):
    wl = _wl([300, 0, 40, 777, 2100], 8, 4, 64, 32, 16, 64, 8, seed=41)
    x = wl.generate(device="cuda")
    cu = x["cu_seqlens"]
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, cu)
    cuc = nsa.nsa_compress_out_len(cu, wl.l, wl.d)
    ncs = [int(n) for n in np.diff(np.concatenate([[0], cuc]))]
    npg = [-(-n // page_size) for n in ncs]
    total = sum(npg) + 2
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(page_size)).to(torch.int32)
    table = torch.full((len(ncs), max(npg) + 1), -1, dtype=torch.int32)
    o = 0
    for b, n in enumerate(npg):
        table[b, :n] = perm[o:o + n]
        o += n
    kp = torch.zeros(total, page_size, wl.n2, wl.d1, dtype=kc.dtype, device="cuda")
    vp = torch.zeros_like(kp)
    nsa.nsa_compress_paged(x["k"], x["v"], x["w"], wl.l, wl.d, cu, kp, vp, table.cuda())
    assert nsa.nsa_compress_status() == 0
    assert torch.equal(_gather(kp.cpu(), table, ncs).view(torch.int16), kc.cpu().view(torch.int16))
    assert torch.equal(_gather(vp.cpu(), table, ncs).view(torch.int16), vc.cpu().view(torch.int16))
    # a decode step: only the last block of each sequence, into a pool holding the others
    kp2, vp2 = kp.clone(), vp.clone()
    for b, n in enumerate(ncs):
        if n:
            pg, r = int(table[b, (n - 1) // page_size]), (n - 1) % page_size
            kp2[pg, r] = 0
            vp2[pg, r] = 0
    nsa.nsa_compress_paged(x["k"], x["v"], x["w"], wl.l, wl.d, cu, kp2, vp2, table.cuda(),
                           first_block=[max(0, n - 1) for n in ncs])
    assert nsa.nsa_compress_status() == 0
    assert torch.equal(kp2, kp) and torch.equal(vp2, vp)


def test_paged_compress_reports_out_of_pool_pages(nsa):
    wl = _wl([900], 8, 2, 64, 32, 16, 64, 8, seed=42)   # 55 blocks: pages 0..3
    x = wl.generate(device="cuda")
    kp = torch.zeros(4, 16, wl.n2, wl.d1, dtype=x["k"].dtype, device="cuda")
    table = torch.tensor([[0, 1, 2, 99]], dtype=torch.int32, device="cuda")   # blocks 48..54 -> page 99: outside
    nsa.nsa_compress_paged(x["k"], None, x["w"], wl.l, wl.d, x["cu_seqlens"], kp, None, table)
    assert nsa.nsa_compress_status() == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_compress_status() == 0                                      # reported once
