"""Pins of the backward oracle (gradient of attention_out with respect to q,
kcmp, vcmp; gradient of the compression with respect to x and w) against
references other than itself: central finite differences of the forward
oracle, float64 torch.autograd of an independent torch restatement, GQA
against replicated heads, and the explicit matrix of the linear compression."""
import numpy as np
import torch

import oracle

L_, D_, LP_ = 8, 4, 8


def _case(lens=(40,), n1=4, n2=2, d1=5, d2=3, seed=0):
    rng = np.random.default_rng(seed)
    ncs = [(s - L_) // D_ + 1 if s >= L_ else 0 for s in lens]
    nss = [-(-s // LP_) for s in lens]
    q = rng.standard_normal((sum(lens), n1, d1))
    kc = rng.standard_normal((sum(ncs), n2, d1))
    vc = rng.standard_normal((sum(ncs), n2, d2))
    return q, kc, vc, np.cumsum(lens), np.cumsum(ncs), np.cumsum(nss)


def _loss(q, kc, vc, R, cq, cc, cs, scale, am=None):
    r = oracle.compress_attention(q, kc, vc, scale, L_, D_, LP_, 2, cq, cc, cs, atten_mask=am)
    return float((r["out"] * R).sum())


def test_attention_backward_matches_finite_differences():
    q, kc, vc, cq, cc, cs = _case(lens=(40, 23))
    rng = np.random.default_rng(1)
    R = rng.standard_normal((q.shape[0], q.shape[1], vc.shape[2]))
    am = rng.random((40, 9)) < 0.25
    for mask in (None, am):
        g = oracle.compress_attention_backward(q, kc, vc, R, 0.7, L_, D_, cq, cc, atten_mask=mask)
        h = 1e-6
        for name, arr, grad in (("q", q, g["dq"]), ("kc", kc, g["dkcmp"]), ("vc", vc, g["dvcmp"])):
            flat = arr.reshape(-1)
            for idx in rng.choice(flat.size, size=12, replace=False):
                keep = flat[idx]
                flat[idx] = keep + h
                up = _loss(q, kc, vc, R, cq, cc, cs, 0.7, mask)
                flat[idx] = keep - h
                dn = _loss(q, kc, vc, R, cq, cc, cs, 0.7, mask)
                flat[idx] = keep
                num = (up - dn) / (2 * h)
                assert abs(num - grad.reshape(-1)[idx]) <= 1e-7 * max(1.0, abs(num)), (name, idx, num)


def _torch_forward(q, kc, vc, cq, cc, scale, am=None):
    """An independent float64 torch restatement of steps 1-3 (causal block mask)."""
    n1, n2 = q.shape[1], kc.shape[1]
    G = n1 // n2
    outs, q0, c0 = [], 0, 0
    for b in range(len(cq)):
        Sq, nc = int(cq[b]) - q0, int(cc[b]) - c0
        qs = q[q0:q0 + Sq]
        if nc == 0:
            outs.append(torch.zeros(Sq, n1, vc.shape[2], dtype=torch.float64))
            q0, c0 = int(cq[b]), int(cc[b])
            continue
        off = max(0, (nc - 1) * D_ + L_ - Sq)
        t = torch.arange(Sq)[:, None] + off
        vis = torch.arange(nc)[None, :] * D_ + L_ - 1 <= t
        if am is not None:
            vis = vis & ~torch.as_tensor(am[:Sq, :nc])
        k = kc[c0:c0 + nc].repeat_interleave(G, dim=1)
        v = vc[c0:c0 + nc].repeat_interleave(G, dim=1)
        s = torch.einsum("thd,ihd->hti", qs, k) * scale
        s = s.masked_fill(~vis[None], float("-inf"))
        p = torch.softmax(s, dim=-1)
        p = torch.nan_to_num(p, nan=0.0)            # rows with no block
        outs.append(torch.einsum("hti,ihd->thd", p, v))
        q0, c0 = int(cq[b]), int(cc[b])
    return torch.cat(outs, 0)


def test_attention_backward_matches_torch_autograd():
    q, kc, vc, cq, cc, cs = _case(lens=(60, 9, 33), n1=6, n2=2, d1=4, d2=6, seed=2)
    rng = np.random.default_rng(3)
    R = rng.standard_normal((q.shape[0], 6, 6))
    am = rng.random((60, 14)) < 0.3
    for mask in (None, am):
        tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, kc, vc))
        (_torch_forward(tq, tk, tv, cq, cc, 0.4, mask) * torch.tensor(R)).sum().backward()
        g = oracle.compress_attention_backward(q, kc, vc, R, 0.4, L_, D_, cq, cc, atten_mask=mask)
        assert np.allclose(g["dq"], tq.grad.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(g["dkcmp"], tk.grad.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(g["dvcmp"], tv.grad.numpy(), rtol=0, atol=1e-12)


def test_gqa_gradients_are_sums_over_replicated_heads():
    q, kc, vc, cq, cc, cs = _case(lens=(50,), n1=4, n2=1, seed=4)
    R = np.random.default_rng(5).standard_normal((50, 4, 3))
    g = oracle.compress_attention_backward(q, kc, vc, R, 0.5, L_, D_, cq, cc)
    g4 = oracle.compress_attention_backward(q, np.repeat(kc, 4, axis=1), np.repeat(vc, 4, axis=1), R, 0.5, L_, D_,
                                            cq, cc)
    assert np.allclose(g["dq"], g4["dq"], rtol=0, atol=1e-13)
    assert np.allclose(g["dkcmp"][:, 0], g4["dkcmp"].sum(axis=1), rtol=0, atol=1e-13)
    assert np.allclose(g["dvcmp"][:, 0], g4["dvcmp"].sum(axis=1), rtol=0, atol=1e-13)


def test_rows_without_blocks_have_no_gradient():
    q, kc, vc, cq, cc, cs = _case(lens=(30,), seed=6)
    R = np.ones((30, 4, 3))
    g = oracle.compress_attention_backward(q, kc, vc, R, 0.5, L_, D_, cq, cc)
    assert (g["dq"][:L_ - 1] == 0).all()            # rows t < l - 1 see no block


def test_compress_backward_is_the_transpose_of_the_linear_map():
    lens, n2, dim, l, d = (21, 8, 30), 2, 3, 8, 4
    rng = np.random.default_rng(7)
    x = rng.standard_normal((sum(lens), n2, dim))
    w = rng.standard_normal((l, n2))
    cu = np.cumsum(lens)
    out, cuc = oracle.compress(x, w, l, d, cu)
    g = rng.standard_normal(out.shape)
    dx, dw = oracle.compress_backward(x, w, g, l, d, cu)
    # explicit matrix of x -> out per head (columns: raw rows, rows: blocks)
    T, Tc = x.shape[0], out.shape[0]
    s0, c0 = 0, 0
    A = np.zeros((n2, Tc, T))
    for s in lens:
        nc = (s - l) // d + 1 if s >= l else 0
        for i in range(nc):
            for j in range(l):
                A[:, c0 + i, s0 + i * d + j] = w[j]
        s0, c0 = s0 + s, c0 + nc
    for n in range(n2):
        assert np.allclose(dx[:, n], A[n].T @ g[:, n], rtol=0, atol=1e-12)
    # dw by central differences of the (unrounded) forward compression
    for j in range(l):
        for n in range(n2):
            wp, wm = w.copy(), w.copy()
            wp[j, n] += 1e-6
            wm[j, n] -= 1e-6
            num = ((oracle.compress(x, wp, l, d, cu)[0] - oracle.compress(x, wm, l, d, cu)[0]) * g).sum() / 2e-6
            assert abs(num - dw[j, n]) <= 1e-6 * max(1.0, abs(num))
