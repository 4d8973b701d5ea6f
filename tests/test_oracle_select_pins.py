"""Pins of the selection-attention oracle (block-sparse attention over the KV
blocks listed per query row and KV group; "lite_boost.ops.rain_fusion_attention",
fed with the top-k of the compressed branch) against references other than
itself: torch's scaled_dot_product_attention and logsumexp in float64 with an
explicit mask, GQA against replicated heads, and the set and alignment
readings checked by self-consistency."""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, mask):
    """q (Sq, N1, D1), k (Skv, N2, D1), v (Skv, N2, D2), mask (Sq, N2, Skv) bool."""
    G = q.shape[1] // k.shape[1]
    qt = torch.tensor(q).permute(1, 0, 2)
    kt = torch.tensor(np.repeat(k, G, axis=1)).permute(1, 0, 2)
    vt = torch.tensor(np.repeat(v, G, axis=1)).permute(1, 0, 2)
    mt = torch.tensor(np.repeat(mask, G, axis=1)).permute(1, 0, 2)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=scale)
    s = (qt @ kt.transpose(1, 2)) * scale
    lse = torch.logsumexp(s.masked_fill(~mt, float("-inf")), dim=-1)
    return out.permute(1, 0, 2).numpy(), lse.T.numpy()


def _case(S=100, n1=4, n2=2, d1=16, d2=8, lp=16, seed=0):
    q = _rand((S, n1, d1), seed)
    k = _rand((S, n2, d1), seed + 1)
    v = _rand((S, n2, d2), seed + 2)
    return q, k, v


def test_all_blocks_listed_is_causal_attention():
    S, lp = 100, 16
    q, k, v = _case(S=S, lp=lp)
    nblk = (S + lp - 1) // lp
    count = nblk + 1
    sel = np.full((S, 2, count), -1, np.int32)
    sel[:, :, :nblk] = np.arange(nblk)
    r = oracle.select_attention(q, k, v, sel, 0.3, lp, count, [S], [S])
    mask = np.tril(np.ones((S, S), bool))[:, None, :].repeat(2, axis=1)
    out, lse = _sdpa(q, k, v, 0.3, mask)
    assert np.allclose(r["out"], out, atol=1e-12)
    assert np.allclose(r["lse"], lse, atol=1e-12)


def test_one_block_per_row_matches_masked_attention():
    S, lp, n2 = 90, 16, 2
    q, k, v = _case(S=S, lp=lp, n2=n2, seed=3)
    rng = np.random.default_rng(7)
    sel = np.full((S, n2, 4), -1, np.int32)
    mask = np.zeros((S, n2, S), bool)
    for t in range(S):
        for g in range(n2):
            j = rng.integers(0, t // lp + 1)
            sel[t, g, 0] = j
            mask[t, g, j * lp:min((j + 1) * lp, t + 1)] = True
    r = oracle.select_attention(q, k, v, sel, 0.25, lp, 4, [S], [S])
    out, lse = _sdpa(q, k, v, 0.25, mask)
    assert np.allclose(r["out"], out, atol=1e-12)
    assert np.allclose(r["lse"], lse, atol=1e-12)


def test_empty_list_gives_zero_output_and_minus_inf():
    q, k, v = _case(S=40)
    sel = np.full((40, 2, 3), -1, np.int32)
    sel[10:, :, 0] = 5          # block 5 starts at 80 > S: past the sequence, ignored
    r = oracle.select_attention(q, k, v, sel, 0.3, 16, 3, [40], [40])
    assert (r["out"] == 0).all()
    assert np.isneginf(r["lse"]).all()


def test_future_block_only_is_empty():
    # block 2 (keys 32..47) lies after query rows 0..31: nothing visible
    q, k, v = _case(S=64)
    sel = np.full((64, 2, 1), 2, np.int32)
    r = oracle.select_attention(q, k, v, sel, 0.3, 16, 1, [64], [64])
    assert np.isneginf(r["lse"][:32]).all() and (r["out"][:32] == 0).all()
    assert np.isfinite(r["lse"][32:]).all()


def test_gqa_equals_replicated_heads():
    S, lp = 70, 16
    q, k, v = _case(S=S, n1=6, n2=2, lp=lp, seed=11)
    rng = np.random.default_rng(1)
    sel = np.sort(rng.integers(0, 5, size=(S, 2, 3)).astype(np.int32), axis=-1)
    r = oracle.select_attention(q, k, v, sel, 0.2, lp, 3, [S], [S])
    k6, v6, sel6 = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), np.repeat(sel, 3, axis=1)
    r6 = oracle.select_attention(q, k6, v6, sel6, 0.2, lp, 3, [S], [S])
    assert np.allclose(r["out"], r6["out"], atol=1e-14)
    assert np.allclose(r["lse"], r6["lse"], atol=1e-14)


def test_list_is_a_set():
    # order, repeats, -1 holes and blocks past the end change nothing
    S, lp = 80, 16
    q, k, v = _case(S=S, seed=5)
    base = np.full((S, 2, 6), -1, np.int32)
    base[:, :, :3] = [0, 2, 4]
    messy = np.full((S, 2, 6), -1, np.int32)
    messy[:, :, :] = [4, -1, 2, 2, 9, 0]
    a = oracle.select_attention(q, k, v, base, 0.3, lp, 6, [S], [S])
    b = oracle.select_attention(q, k, v, messy, 0.3, lp, 6, [S], [S])
    # (the key order differs, so the sums agree up to rounding order)
    assert np.allclose(a["out"], b["out"], rtol=0, atol=1e-13)
    assert np.allclose(a["lse"], b["lse"], rtol=0, atol=1e-13)


def test_short_queries_are_bottom_right_aligned():
    S, Sq, lp = 96, 20, 16
    q, k, v = _case(S=S, seed=9)
    rng = np.random.default_rng(2)
    sel = np.sort(rng.integers(0, 6, size=(S, 2, 4)).astype(np.int32), axis=-1)
    full = oracle.select_attention(q, k, v, sel, 0.3, lp, 4, [S], [S])
    short = oracle.select_attention(q[S - Sq:], k, v, sel[S - Sq:], 0.3, lp, 4, [Sq], [S])
    assert np.array_equal(short["out"], full["out"][S - Sq:])
    assert np.array_equal(short["lse"], full["lse"][S - Sq:])


def test_varlen_sequences_are_independent_and_rows_sample():
    lens_q, lens_kv, lp = [30, 1, 45], [50, 16, 45], 16
    cq, ck = np.cumsum(lens_q).astype(np.int32), np.cumsum(lens_kv).astype(np.int32)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((cq[-1], 4, 8))
    k = rng.standard_normal((ck[-1], 2, 8))
    v = rng.standard_normal((ck[-1], 2, 8))
    sel = np.sort(rng.integers(-1, 4, size=(cq[-1], 2, 3)).astype(np.int32), axis=-1)
    sel = np.concatenate([np.sort(np.where(sel >= 0, sel, 1 << 20), axis=-1)], axis=0)
    sel[sel == 1 << 20] = -1
    allr = oracle.select_attention(q, k, v, sel, 0.4, lp, 3, cq, ck)
    q0, k0 = 0, 0
    for b in range(3):
        one = oracle.select_attention(q[q0:cq[b]], k[k0:ck[b]], v[k0:ck[b]], sel[q0:cq[b]], 0.4, lp, 3,
                                      [lens_q[b]], [lens_kv[b]])
        assert np.array_equal(one["out"], allr["out"][q0:cq[b]])
        q0, k0 = cq[b], ck[b]
    rows = np.array([0, 29, 30, 31, 75], dtype=np.int64)
    samp = oracle.select_attention(q[rows], k, v, sel, 0.4, lp, 3, cq, ck, rows=rows, q_rows_only=True)
    assert np.array_equal(samp["out"], allr["out"][rows])


def test_closed_form_two_keys():
    # q = (1, 0); k_0 = (1, 0), k_1 = (0, 1); v_0 = (1, 0), v_1 = (0, 2); scale 1;
    # blocks of one key, row 1 lists both: weights e/(e+1), 1/(e+1)
    q = np.array([[[0.0, 0.0]], [[1.0, 0.0]]])
    k = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    v = np.array([[[1.0, 0.0]], [[0.0, 2.0]]])
    sel = np.array([[[0, -1]], [[0, 1]]], np.int32)
    r = oracle.select_attention(q, k, v, sel, 1.0, 1, 2, [2], [2])
    e = np.e
    assert np.allclose(r["out"][1, 0], [e / (e + 1), 2 / (e + 1)], rtol=0, atol=1e-15)
    assert abs(r["lse"][1, 0] - np.log(e + 1)) < 1e-15
    # row 0 sees only key 0: the output is v_0, the lse its scaled score (0)
    assert np.array_equal(r["out"][0, 0], [1.0, 0.0]) and r["lse"][0, 0] == 0.0


def test_closed_form_causal_cut_inside_a_block():
    # one block of 4 keys; row t sees keys 0..t: with equal scores the output
    # is the mean of the first t+1 value rows and the lse is log(t+1)
    S = 4
    q = np.zeros((S, 1, 2))
    k = np.zeros((S, 1, 2))
    v = np.arange(S, dtype=np.float64).reshape(S, 1, 1) * np.ones((1, 1, 2))
    sel = np.zeros((S, 1, 1), np.int32)
    r = oracle.select_attention(q, k, v, sel, 0.7, 4, 1, [S], [S])
    for t in range(S):
        assert np.allclose(r["out"][t, 0], np.full(2, t / 2.0), rtol=0, atol=1e-15)
        assert abs(r["lse"][t, 0] - np.log(t + 1)) < 1e-15
