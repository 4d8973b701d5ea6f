"""Parity of nsa_compress_attention with the page's optional masks
(atten_mask at step 1, topk_mask at step 6; True removes the pair, one (S1, S2)
matrix for every sequence and head, row = query index inside the sequence)
against the fp64 oracle given the same masks and the same storage-dtype
kcmp / vcmp."""
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


def _wl(seqs, n1, n2, dd, l, d, lp, count, seed=7, dtype="bf16"):
    return workloads.Workload("case", tuple(seqs), n1, n2, dd, dd, l, d, lp, count, dd ** -0.5, dtype, seed=seed)


def _inputs(wl, device="cpu"):
    x = wl.generate(device=device)
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    return x, torch.from_numpy(kc).to(wl.torch_dtype), torch.from_numpy(vc).to(wl.torch_dtype), cuc


def _masks(wl, x, cuc, p_att, p_topk, seed):
    rng = np.random.default_rng(seed)
    sq = np.diff(np.concatenate([[0], x["cu_seqlens_q"]]))
    nc = np.diff(np.concatenate([[0], cuc]))
    ns = np.diff(np.concatenate([[0], x["cu_sel_kv"]]))
    am = rng.random((int(sq.max()), max(1, int(nc.max())))) < p_att if p_att is not None else None
    tm = rng.random((int(sq.max()), max(1, int(ns.max())))) < p_topk if p_topk is not None else None
    return am, tm


def _gpu(nsa, wl, x, kc, vc, cuc, am, tm):
    ws = torch.empty(nsa.nsa_compress_attention_masked_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"],
        am is not None, tm is not None), dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention(
        x["q"].cuda(), kc.cuda(), vc.cuda(), wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
        x["cu_sel_kv"], workspace=ws,
        atten_mask=torch.from_numpy(am).cuda() if am is not None else None,
        topk_mask=torch.from_numpy(tm).cuda() if tm is not None else None)
    assert nsa.nsa_workspace_status(ws) == 0
    return [t.cpu() for t in res]


def _check(res, ref, wl, x, tm, rows=None, tie_rel=1e-4):
    att, tk, smax, ssum = res
    rows = ref["rows"] if rows is None else rows
    g_out = att.double().numpy()[rows]
    assert np.isfinite(g_out).all()
    assert np.abs(g_out - ref["out"]).max() <= 1e-2
    gm, gs = smax.numpy()[rows][..., 0].astype(np.float64), ssum.numpy()[rows][..., 0].astype(np.float64)
    empty = np.isneginf(ref["softmax_max"])
    assert (np.isneginf(gm) == empty).all() and (gs[empty] == 0).all()
    for g, r in ((gm[~empty], ref["softmax_max"][~empty]), (gs[~empty], ref["softmax_sum"][~empty])):
        denom = np.where(np.abs(r) < 1e-3, 1.0, np.abs(r))
        assert (np.abs(g - r) <= 1e-3 * denom + np.where(np.abs(r) < 1e-3, 1e-6, 0)).all()
    cq = x["cu_seqlens_q"]
    cs = x["cu_sel_kv"]
    g_tk = tk.numpy()[rows]
    for ri, row in enumerate(rows):
        b = int(np.searchsorted(cq, row, side="right"))
        tloc = row - (int(cq[b - 1]) if b else 0)
        # the row's position t (query offset of the sequence, as in step 1's
        # causal rule) and its selection-block count: a causal candidate j has
        # j < n_sel and j * l' <= t
        s_raw = wl.seqlens[b]
        n_cmp = 0 if s_raw < wl.l else (s_raw - wl.l) // wl.d + 1
        s_q = int(cq[b]) - (int(cq[b - 1]) if b else 0)
        t_pos = tloc + (max(0, (n_cmp - 1) * wl.d + wl.l - s_q) if n_cmp else 0)
        n_sel = int(cs[b]) - (int(cs[b - 1]) if b else 0)
        for g in range(wl.n2):
            a, r = g_tk[ri, g], ref["topk"][ri, g]
            na, nr = int((a >= 0).sum()), int((r >= 0).sum())
            assert na == nr and (a[na:] == -1).all(), (row, g, a, r)
            va, vr = a[:na], r[:nr]
            if na == 0:
                continue
            assert (np.diff(va) > 0).all()
            assert va.min() >= 0 and va.max() < n_sel, f"row {row} group {g}: index past the sequence {va}"
            assert (va.astype(np.int64) * wl.lp <= t_pos).all(), f"row {row} group {g}: future block in {va}"
            if tm is not None:
                assert not tm[tloc, va].any(), "a masked candidate was selected"
            if set(va.tolist()) != set(vr.tolist()):
                sc = ref["score"][ri, g]
                kth = np.sort(sc[vr])[0]
                for j in set(va.tolist()) ^ set(vr.tolist()):
                    assert abs(sc[j] - kth) <= tie_rel * abs(kth), (row, g, j, sc[j], kth)


@pytest.mark.parametrize("l,d,lp", [(32, 16, 64), (32, 16, 32), (16, 16, 128), (64, 32, 64)],
                         ids=["a4", "a2", "a8", "a2_l64"])
def test_random_masks(nsa, l, d, lp):
    wl = _wl([1500], 16, 2, 64, l, d, lp, 6, seed=21)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.3, 0.3, seed=1)
    res = _gpu(nsa, wl, x, kc, vc, cuc, am, tm)
    ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"], atten_mask=am, topk_mask=tm)
    _check(res, ref, wl, x, tm)


@pytest.mark.parametrize("l,d,lp", [(32, 16, 64), (32, 16, 32)], ids=["a4", "a2"])
def test_masks_wider_than_the_blocks(nsa, l, d, lp):
    # mask rows longer than the blocks of any sequence (padded to a multiple
    # of 16 bytes); the extra columns are set and must be ignored
    wl = _wl([1300, 200], 16, 2, 64, l, d, lp, 6, seed=25)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.3, 0.3, seed=6)
    pad = lambda m_: np.concatenate([m_, np.ones((m_.shape[0], -m_.shape[1] % 16 or 16), bool)], axis=1)
    am, tm = pad(am), pad(tm)
    assert am.shape[1] % 16 == 0 and tm.shape[1] % 16 == 0
    res = _gpu(nsa, wl, x, kc, vc, cuc, am, tm)
    ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"], atten_mask=am, topk_mask=tm)
    _check(res, ref, wl, x, tm)


def test_one_mask_at_a_time_and_fully_masked_rows(nsa):
    wl = _wl([900], 8, 2, 64, 32, 16, 64, 5, seed=22)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.2, 0.5, seed=2)
    am[300:340] = True                       # rows that end up attending to nothing
    for a_, t_ in ((am, None), (None, tm)):
        res = _gpu(nsa, wl, x, kc, vc, cuc, a_, t_)
        ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                        x["cu_seqlens_q"], cuc, x["cu_sel_kv"], atten_mask=a_, topk_mask=t_)
        _check(res, ref, wl, x, t_)
    assert np.isneginf(ref["softmax_max"][300:340]).sum() == 0   # topk_mask alone leaves them
    res = _gpu(nsa, wl, x, kc, vc, cuc, am, None)
    assert (res[1].numpy()[300:340] == -1).all() and (res[0].float().numpy()[300:340] == 0).all()


def test_varlen_shares_one_mask(nsa):
    wl = _wl([300, 0, 40, 777], 16, 4, 64, 32, 16, 64, 8, seed=23)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.25, 0.25, seed=3)
    res = _gpu(nsa, wl, x, kc, vc, cuc, am, tm)
    ref = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"], atten_mask=am, topk_mask=tm)
    _check(res, ref, wl, x, tm)


def test_all_false_masks_equal_the_unmasked_kernel(nsa):
    wl = _wl([2000], 32, 2, 128, 32, 16, 64, 16, seed=24)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.0, 0.0, seed=4)
    masked = _gpu(nsa, wl, x, kc, vc, cuc, am, tm)
    plain = _gpu(nsa, wl, x, kc, vc, cuc, None, None)
    for a, b in zip(masked, plain):
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.int32 else a,
                           b.view(torch.uint8) if b.dtype != torch.int32 else b)


def test_masks_on_the_16k_workload_sampled_rows(nsa):
    wl = workloads.SINGLE_16K
    x = wl.generate(device="cuda")
    cuc = nsa.nsa_compress_out_len(x["cu_seqlens"], wl.l, wl.d)
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"])
    am, tm = _masks(wl, x, cuc, 0.3, 0.3, seed=5)
    ws = torch.empty(nsa.nsa_compress_attention_masked_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
        dtype=torch.uint8, device="cuda")
    res = nsa.nsa_compress_attention(x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                     x["cu_seqlens_q"], cuc, x["cu_sel_kv"], workspace=ws,
                                     atten_mask=torch.from_numpy(am).cuda(), topk_mask=torch.from_numpy(tm).cuda())
    assert nsa.nsa_workspace_status(ws) == 0
    rows = workloads.sample_rows(x["cu_seqlens_q"], first=64, last=64, every=331)
    rows_t = torch.from_numpy(rows).cuda()
    ref = oracle.compress_attention(x["q"].index_select(0, rows_t).float().cpu(), kc.float().cpu(),
                                    vc.float().cpu(), wl.scale, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc,
                                    x["cu_sel_kv"], rows=rows, q_rows_only=True, atten_mask=am, topk_mask=tm)
    _check([t.cpu() for t in res], ref, wl, x, tm)


def test_masked_call_needs_the_masked_workspace(nsa):
    wl = _wl([700], 8, 2, 64, 32, 16, 64, 5, seed=26)
    x, kc, vc, cuc = _inputs(wl)
    am, tm = _masks(wl, x, cuc, 0.3, 0.3, seed=7)
    small = nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    need = nsa.nsa_compress_attention_masked_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    assert need > small
    with pytest.raises(ValueError):
        nsa.nsa_compress_attention(x["q"].cuda(), kc.cuda(), vc.cuda(), wl.scale, wl.n1, wl.l, wl.d, wl.lp,
                                   wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"],
                                   workspace=torch.empty(small, dtype=torch.uint8, device="cuda"),
                                   atten_mask=torch.from_numpy(am).cuda(), topk_mask=torch.from_numpy(tm).cuda())
