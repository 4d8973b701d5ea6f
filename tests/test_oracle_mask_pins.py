"""Pins of the optional masks of mindspore.ops.nsa_compress_attention in the
oracle (description step 1: QK = atten_mask(QK, atten_mask); step 6:
P'_slc = topk_mask(P'_slc); keyword arguments atten_mask (S1, S2cmp) and
topk_mask (S1, S2sel), bool).  Reading: True removes the (query, block) pair;
one matrix serves every sequence and head, indexed by the query index inside
its sequence.  References: float64 SDPA with the combined causal-and-mask
pattern, identities with the unmasked oracle, and torch.sort for the top-k."""
import numpy as np
import torch

import oracle

L_, D_, LP_ = 32, 16, 64


def _case(S=300, n1=4, n2=2, dd=16, seed=0):
    rng = np.random.default_rng(seed)
    n_cmp = (S - L_) // D_ + 1
    q = rng.standard_normal((S, n1, dd))
    kc = rng.standard_normal((n_cmp, n2, dd))
    vc = rng.standard_normal((n_cmp, n2, dd))
    n_sel = -(-S // LP_)
    return q, kc, vc, n_cmp, n_sel


def _run(q, kc, vc, S, n_cmp, n_sel, count=3, **kw):
    return oracle.compress_attention(q, kc, vc, 0.25, L_, D_, LP_, count, [S], [n_cmp], [n_sel], **kw)


def test_all_false_masks_change_nothing():
    S = 300
    q, kc, vc, nc, ns = _case(S)
    a = _run(q, kc, vc, S, nc, ns)
    b = _run(q, kc, vc, S, nc, ns, atten_mask=np.zeros((S, nc), bool), topk_mask=np.zeros((S, ns), bool))
    for key in ("out", "softmax_max", "softmax_sum", "topk", "score"):
        assert np.array_equal(a[key], b[key]), key


def test_masking_only_future_blocks_changes_nothing():
    S = 300
    q, kc, vc, nc, ns = _case(S, seed=1)
    t = np.arange(S)[:, None]
    future = np.arange(nc)[None, :] * D_ + L_ - 1 > t          # blocks the causal rule hides anyway
    a = _run(q, kc, vc, S, nc, ns)
    b = _run(q, kc, vc, S, nc, ns, atten_mask=future)
    for key in ("out", "softmax_max", "softmax_sum", "topk"):
        assert np.array_equal(a[key], b[key]), key


def test_atten_mask_matches_sdpa_with_the_combined_mask():
    S, n1, n2 = 260, 4, 2
    q, kc, vc, nc, ns = _case(S, n1, n2, seed=2)
    rng = np.random.default_rng(7)
    am = rng.random((S, nc)) < 0.3
    r = _run(q, kc, vc, S, nc, ns, atten_mask=am)
    t = np.arange(S)[:, None]
    keep = (np.arange(nc)[None, :] * D_ + L_ - 1 <= t) & ~am   # (S, nc)
    rows = keep.any(axis=1)
    G = n1 // n2
    qt = torch.tensor(q).permute(1, 0, 2)
    kt = torch.tensor(np.repeat(kc, G, axis=1)).permute(1, 0, 2)
    vt = torch.tensor(np.repeat(vc, G, axis=1)).permute(1, 0, 2)
    mt = torch.tensor(keep)[None].expand(n1, S, nc)
    s = (qt @ kt.transpose(1, 2)) * 0.25
    ref = torch.nn.functional.scaled_dot_product_attention(qt[:, rows], kt, vt, attn_mask=mt[:, rows], scale=0.25)
    lse = torch.logsumexp(s.masked_fill(~mt, float("-inf")), dim=-1).T.numpy()
    assert np.allclose(r["out"][rows], ref.permute(1, 0, 2).numpy(), atol=1e-12)
    got = r["softmax_max"][rows] + np.log(r["softmax_sum"][rows])
    assert np.allclose(got, lse[rows], atol=1e-12)
    # rows left without a block: empty-row outputs
    assert (~rows).any()
    assert (r["out"][~rows] == 0).all() and np.isneginf(r["softmax_max"][~rows]).all()
    assert (r["softmax_sum"][~rows] == 0).all() and (r["topk"][~rows] == -1).all()


def test_masked_importance_matches_convolution_of_the_masked_softmax():
    # P of a row restricted to its kept blocks (numpy softmax), then the band of
    # step 4 as two box convolutions sampled at a*j, summed over the group
    S, n1, n2 = 400, 4, 2
    q, kc, vc, nc, ns = _case(S, n1, n2, seed=3)
    rng = np.random.default_rng(11)
    am = rng.random((S, nc)) < 0.25
    r = _run(q, kc, vc, S, nc, ns, atten_mask=am)
    a, bb, G = LP_ // D_, L_ // D_, n1 // n2
    for t in range(0, S, 13):
        keep = (np.arange(nc) * D_ + L_ - 1 <= t) & ~am[t]
        if not keep.any():
            continue
        nvis = int((np.arange(nc) * D_ + L_ - 1 <= t).sum())
        for g in range(n2):
            want = np.zeros(ns)
            for hh in range(G):
                h = g * G + hh
                sc = 0.25 * (kc[:, g] @ q[t, h])
                x = np.where(keep, sc, -np.inf)
                P = np.exp(x - x.max())
                P = (P / P.sum())[:nvis]
                c = np.convolve(np.convolve(P, np.ones(a)), np.ones(bb))
                want += np.array([c[a * j] if a * j < c.size else 0.0 for j in range(ns)])
            assert np.allclose(r["score"][t, g, :ns], want, rtol=0, atol=1e-12)


def test_topk_mask_is_torch_sort_over_the_remaining_candidates():
    S = 900
    q, kc, vc, nc, ns = _case(S, seed=4)
    rng = np.random.default_rng(9)
    tm = rng.random((S, ns)) < 0.4
    count = 4
    r = _run(q, kc, vc, S, nc, ns, count=count, topk_mask=tm)
    base = _run(q, kc, vc, S, nc, ns, count=count)
    assert np.array_equal(r["score"], base["score"])          # the mask acts after the scores
    for row in range(0, S, 7):
        for g in range(kc.shape[1]):
            if r["ncand"][row, g] == 0 and base["ncand"][row, g] == 0:
                continue
            ncand = min(ns, row // LP_ + 1)
            cand = [j for j in range(ncand) if not tm[row, j]]
            sc = torch.tensor(r["score"][row, g, cand])
            order = torch.sort(-sc, stable=True).indices[:count].tolist()
            want = sorted(cand[i] for i in order)
            want += [-1] * (count - len(want))
            assert r["topk"][row, g].tolist() == want


def test_masks_are_indexed_by_the_query_inside_its_sequence():
    lens = [200, 130]
    rng = np.random.default_rng(5)
    n1, n2, dd = 4, 2, 16
    ncs = [(s - L_) // D_ + 1 for s in lens]
    nss = [-(-s // LP_) for s in lens]
    q = rng.standard_normal((sum(lens), n1, dd))
    kc = rng.standard_normal((sum(ncs), n2, dd))
    vc = rng.standard_normal((sum(ncs), n2, dd))
    am = rng.random((max(lens), max(ncs))) < 0.3
    tm = rng.random((max(lens), max(nss))) < 0.3
    cq, cc, cs = np.cumsum(lens), np.cumsum(ncs), np.cumsum(nss)
    both = oracle.compress_attention(q, kc, vc, 0.3, L_, D_, LP_, 3, cq, cc, cs, atten_mask=am, topk_mask=tm)
    q0 = c0 = 0
    for b in range(2):
        one = oracle.compress_attention(q[q0:cq[b]], kc[c0:cc[b]], vc[c0:cc[b]], 0.3, L_, D_, LP_, 3,
                                        [lens[b]], [ncs[b]], [nss[b]], atten_mask=am, topk_mask=tm)
        for key in ("out", "topk", "softmax_sum"):
            assert np.array_equal(one[key], both[key][q0:cq[b]]), key
        q0, c0 = cq[b], cc[b]


def test_closed_form_equal_scores_under_a_mask():
    # q = 0: every visible score is 0, so a row's output is the mean of its
    # visible, unmasked value blocks, softmax_max = 0 and softmax_sum = their count
    S, n1, n2, dd = 200, 2, 1, 4
    n_cmp = (S - L_) // D_ + 1
    n_sel = -(-S // LP_)
    q = np.zeros((S, n1, dd))
    kc = np.random.default_rng(0).standard_normal((n_cmp, n2, dd))
    vc = np.arange(n_cmp, dtype=np.float64)[:, None, None] * np.ones((1, n2, dd))
    am = np.zeros((S, n_cmp), bool)
    am[:, 1::3] = True                     # every third block from 1 on
    r = oracle.compress_attention(q, kc, vc, 0.5, L_, D_, LP_, 2, [S], [n_cmp], [n_sel], atten_mask=am)
    for t in range(S):
        kept = [i for i in range(n_cmp) if i * D_ + L_ - 1 <= t and not am[t, i]]
        if not kept:
            assert np.isneginf(r["softmax_max"][t]).all() and (r["out"][t] == 0).all()
            continue
        assert np.allclose(r["out"][t], np.mean(kept), rtol=0, atol=1e-12)
        assert (r["softmax_max"][t] == 0).all() and np.allclose(r["softmax_sum"][t], len(kept), atol=1e-12)
