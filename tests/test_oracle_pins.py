"""Pins of the fp64 oracle against things other than itself.

Each test ties one step of the oracle to a hand-worked example (tests/golden),
a closed form, an invariant, a special case that reduces to a library routine
(torch / numpy), or brute force on a tiny case.  Together they are chosen so
that a dropped term, a wrong sign or index, or a transposed operand in any
step of the oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from conftest import read_golden


# --------------------------------------------------------------------------
# rounding fp64 -> storage dtype (RNE)
# --------------------------------------------------------------------------
def test_round_bf16_matches_torch_on_fp32_values():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(200000, generator=g) * torch.exp(torch.randn(200000, generator=g) * 8)
    # exact halfway points between neighbouring bf16 values, both parities
    base = torch.randn(4096, generator=g).to(torch.bfloat16).float()
    half = base + torch.sign(base) * base.abs() * 2.0 ** -8 * 0.5
    tiny = torch.tensor([1e-40, -3e-39, 2.0 ** -133, 2.0 ** -134 * 3], dtype=torch.float32)
    x = torch.cat([x, half, tiny]).float()
    want = x.to(torch.bfloat16).double().numpy()
    got = oracle.round_storage(x.double().numpy(), oracle.BF16)
    np.testing.assert_array_equal(got, want)


def test_round_fp16_matches_numpy():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(200000) * np.exp(rng.standard_normal(200000) * 4)
    x = np.concatenate([x, [65504.0, 65520.0, 65519.99, 1e-8, 2.0 ** -25, 3 * 2.0 ** -26]])
    want = x.astype(np.float16).astype(np.float64)
    got = oracle.round_storage(x, oracle.FP16)
    np.testing.assert_array_equal(got, want)


# --------------------------------------------------------------------------
# compression (aclnnNsaCompress, Formula section)
# --------------------------------------------------------------------------
def test_compress_golden():
    gd = read_golden("compress_tiny.txt")
    l, d = int(gd["l"][0]), int(gd["d"][0])
    k = np.array(gd["k"][0].split(), dtype=np.float64).reshape(-1, 1, 1)
    w = np.array(gd["w"][0].split(), dtype=np.float64).reshape(-1, 1)
    want = np.array(gd["kcmp"][0].split(), dtype=np.float64)
    out, cu = oracle.compress(k, w, l, d, [k.shape[0]])
    assert cu.tolist() == [len(want)]
    np.testing.assert_array_equal(out.reshape(-1), want)


def test_compress_lengths_of_the_workloads():
    # block counts worked by hand from floor((S - l)/d) + 1
    assert oracle.compress_len([16384], 32, 16).tolist() == [1023]
    assert oracle.compress_len([131072], 64, 32).tolist() == [4095]
    assert oracle.compress_len(np.cumsum([65536] * 4), 128, 64).tolist() == [1023, 2046, 3069, 4092]
    assert oracle.compress_len([1024], 32, 16).tolist() == [63]


def test_compress_lengths_short_and_ragged():
    # S < l gives no block (floor of a negative number, not truncation)
    lens = [31, 0, 32, 33, 47, 48]
    per = np.diff(np.concatenate([[0], oracle.compress_len(np.cumsum(lens), 32, 16)]))
    assert per.tolist() == [0, 0, 1, 1, 1, 2]
    assert oracle.compress_len(np.cumsum([0, 10, 16]), 16, 16).tolist() == [0, 0, 1]


def _raw(S, n2, D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(S, n2, D, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("l,d", [(32, 16), (64, 32), (48, 16), (16, 16), (128, 64)])
def test_compress_one_hot_weight_is_a_copy(l, d):
    seqs = [200, 7, 131]
    x = _raw(sum(seqs), 3, 16, 1)
    cu = np.cumsum(seqs)
    j0 = [0, l // 2, l - 1]
    w = np.zeros((l, 3))
    for n in range(3):
        w[j0[n], n] = 1.0
    out, cuc = oracle.compress(x, w, l, d, cu, dtype=oracle.BF16)
    xf = x.double().numpy()
    starts = np.concatenate([[0], cu[:-1]])
    cstarts = np.concatenate([[0], cuc[:-1]])
    for b in range(len(seqs)):
        for i in range(cuc[b] - cstarts[b]):
            for n in range(3):
                np.testing.assert_array_equal(out[cstarts[b] + i, n], xf[starts[b] + i * d + j0[n], n])


@pytest.mark.parametrize("l,d", [(32, 16), (64, 64), (16, 16), (128, 32)])
def test_compress_uniform_weight_is_window_mean(l, d):
    S = 517
    x = _raw(S, 2, 8, 2).double().numpy()
    w = np.full((l, 2), 1.0 / l)          # l is a power of two: 1/l is exact
    out, cuc = oracle.compress(x, w, l, d, [S])
    win = np.lib.stride_tricks.sliding_window_view(x, l, axis=0)[::d]   # (n, N2, D, l)
    np.testing.assert_allclose(out, win.mean(axis=-1), rtol=0, atol=1e-14)


def test_compress_nonoverlapping_blocks_are_block_sums():
    l = d = 32
    S = 32 * 9 + 5
    x = _raw(S, 2, 8, 3).double().numpy()
    rng = np.random.default_rng(3)
    w = rng.random((l, 2))
    out, cuc = oracle.compress(x, w, l, d, [S])
    blocks = x[:9 * 32].reshape(9, 32, 2, 8)
    want = np.einsum("ijnk,jn->ink", blocks, w)
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# importance score (step 4) and top-k (step 7)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["importance_a2_b2.txt", "importance_a4_b2_uniform.txt"])
def test_importance_golden(name):
    gd = read_golden(name)
    a, b, n_sel = int(gd["a"][0]), int(gd["b"][0]), int(gd["n_sel"][0])
    P = np.array(gd["P"][0].split(), dtype=np.float64)
    want = np.array(gd["P_slc"][0].split(), dtype=np.float64)
    got = oracle.importance(P, len(P), a, b, n_sel)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    count = int(gd["count"][0])
    tk = oracle.topk(got, n_sel, count)
    assert tk.tolist() == [int(x) for x in gd["topk"][0].split()]


@pytest.mark.parametrize("a,b", [(a, b) for a in range(1, 9) for b in range(1, a + 1)])
def test_importance_is_decimated_convolution(a, b):
    """Step 4 equals np.convolve of P with ones(a) * ones(b), sampled at a*j."""
    rng = np.random.default_rng(a * 10 + b)
    n_vis = 37
    P = rng.random(n_vis)
    kern = np.convolve(np.ones(a), np.ones(b))          # multiplicity of each m + n
    full = np.convolve(P, kern)                          # full[c] = sum_u kern[u] P[c-u]
    n_sel = (n_vis + a + b) // a + 2
    want = np.array([full[a * j] if a * j < full.size else 0.0 for j in range(n_sel)])
    got = oracle.importance(P, n_vis, a, b, n_sel)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("a,b", [(2, 2), (4, 2), (4, 4), (3, 1), (8, 5)])
def test_importance_column_sum_invariant(a, b):
    """Every visible P[c] is counted b times over all j when n_sel is large."""
    rng = np.random.default_rng(7)
    P = rng.random(50)
    got = oracle.importance(P, 50, a, b, (50 + a + b) // a + 1)
    assert math.isclose(got.sum(), b * P.sum(), rel_tol=1e-13)


def test_importance_ignores_invisible_blocks():
    P = np.arange(1.0, 11.0)
    got = oracle.importance(P, 6, 2, 2, 6)      # only P[0..5] are visible
    want = oracle.importance(np.concatenate([P[:6], np.zeros(4)]), 10, 2, 2, 6)
    np.testing.assert_array_equal(got, want)


def test_topk_golden_ties_and_padding():
    for case in read_golden("topk_ties.txt")["case"]:
        sc, cnt, want = [s.strip() for s in case.split("|")]
        s = np.array(sc.split(), dtype=np.float64)
        got = oracle.topk(s, len(s), int(cnt))
        assert got.tolist() == [int(x) for x in want.split()]


def test_topk_matches_torch_sort_without_ties():
    rng = np.random.default_rng(5)
    for n_cand in [1, 5, 31, 32, 33, 200, 1024]:
        for count in [1, 8, 16, 32]:
            s = rng.random(n_cand)
            got = oracle.topk(s, n_cand, count)
            k = min(count, n_cand)
            order = torch.sort(torch.from_numpy(s), descending=True, stable=True).indices[:k]
            want = sorted(order.tolist()) + [-1] * (count - k)
            assert got.tolist() == want


# --------------------------------------------------------------------------
# compressed attention (steps 1-3) against library routines
# --------------------------------------------------------------------------
def _small_case(S=300, n1=4, n2=2, d1=32, d2=16, l=32, d=16, lp=64, count=4, seed=11,
                seqs=None):
    seqs = seqs or [S]
    g = torch.Generator().manual_seed(seed)
    T = sum(seqs)
    q = torch.randn(T, n1, d1, generator=g).to(torch.bfloat16)
    kc_n = oracle.compress_len(np.cumsum(seqs), l, d)
    tc = int(kc_n[-1])
    kc = torch.randn(tc, n2, d1, generator=g).to(torch.bfloat16)
    vc = torch.randn(tc, n2, d2, generator=g).to(torch.bfloat16)
    cu_sel = np.cumsum([-(-s // lp) for s in seqs]).astype(np.int32)
    return dict(q=q, kc=kc, vc=vc, l=l, d=d, lp=lp, count=count,
                cu_q=np.cumsum(seqs).astype(np.int32), cu_cmp=kc_n, cu_sel=cu_sel,
                scale=d1 ** -0.5)


def _run(c, **kw):
    return oracle.compress_attention(c["q"], c["kc"], c["vc"], c["scale"], c["l"], c["d"],
                                     c["lp"], c["count"], c["cu_q"], c["cu_cmp"], c["cu_sel"], **kw)


def _mask_single(S, n_cmp, l, d):
    t = np.arange(S)[:, None]
    i = np.arange(n_cmp)[None, :]
    return (i * d + l - 1) <= t


def test_attention_matches_torch_sdpa_float64():
    c = _small_case()
    r = _run(c)
    S, n1, n2 = c["q"].shape[0], c["q"].shape[1], c["kc"].shape[1]
    G = n1 // n2
    mask = torch.from_numpy(_mask_single(S, c["kc"].shape[0], c["l"], c["d"]))
    q = c["q"].double().permute(1, 0, 2)                       # (N1, S, D1)
    k = c["kc"].double().permute(1, 0, 2).repeat_interleave(G, 0)
    v = c["vc"].double().permute(1, 0, 2).repeat_interleave(G, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=mask, scale=c["scale"]).permute(1, 0, 2).numpy()
    rows = mask.any(1).numpy()
    np.testing.assert_allclose(r["out"][rows], ref[rows], rtol=1e-12, atol=1e-12)
    # m + log L equals the log-sum-exp of the masked scaled scores
    sc = torch.einsum("hsd,htd->sht", q.permute(1, 0, 2).permute(1, 0, 2), k) * c["scale"]
    sc = sc.masked_fill(~mask[:, None, :], float("-inf"))
    lse = torch.logsumexp(sc, dim=-1).numpy()
    got = r["softmax_max"] + np.log(r["softmax_sum"])
    np.testing.assert_allclose(got[rows], lse[rows], rtol=1e-12, atol=1e-12)


def test_attention_one_hot_values_expose_softmax_rows():
    """With vcmp[i] = e_i the output row is P itself: rows sum to 1 and equal
    torch.softmax of the masked scores."""
    c = _small_case(S=200, n1=2, n2=1, d1=16, d2=16, l=32, d=16)
    n_cmp = c["kc"].shape[0]
    assert n_cmp <= 16
    vc = torch.zeros(n_cmp, 1, 16)
    vc[torch.arange(n_cmp), 0, torch.arange(n_cmp)] = 1.0
    c["vc"] = vc.to(torch.bfloat16)
    r = _run(c)
    mask = _mask_single(200, n_cmp, 32, 16)
    rows = mask.any(1)
    P = r["out"][:, :, :n_cmp]
    np.testing.assert_allclose(P[rows].sum(-1), 1.0, rtol=0, atol=1e-12)
    sc = torch.einsum("shd,td->sht", c["q"].double(), c["kc"][:, 0].double()) * c["scale"]
    sc = sc.masked_fill(~torch.from_numpy(mask)[:, None, :], float("-inf"))
    want = torch.softmax(sc, -1).numpy()
    np.testing.assert_allclose(P[rows], want[rows], rtol=1e-12, atol=1e-14)
    assert np.all(r["out"][:, :, n_cmp:] == 0)


def test_attention_single_visible_block():
    c = _small_case(S=60, n1=2, n2=1)
    r = _run(c)
    # l = 32, d = 16: t = 31..46 see block 0 only
    q = c["q"].double().numpy()
    k0 = c["kc"].double().numpy()[0, 0]
    for t in range(31, 47):
        for h in range(2):
            np.testing.assert_array_equal(r["out"][t, h], c["vc"].double().numpy()[0, 0])
            assert r["softmax_sum"][t, h] == 1.0
            assert math.isclose(r["softmax_max"][t, h], c["scale"] * float(q[t, h] @ k0),
                                rel_tol=1e-14)


def test_attention_identical_keys_count_visible_blocks():
    """Identical keys give uniform P: softmax_sum counts the visible blocks and
    the output is the mean of the visible values."""
    for (l, d) in [(32, 16), (64, 32), (48, 16), (16, 16)]:
        S = 400
        c = _small_case(S=S, n1=2, n2=1, l=l, d=d, lp=max(64, l))
        n_cmp = c["kc"].shape[0]
        c["kc"] = c["kc"][:1].repeat(n_cmp, 1, 1)
        r = _run(c)
        vc = c["vc"].double().numpy()[:, 0]
        for t in range(S):
            nvis = 0 if t < l - 1 else min(n_cmp, (t - l + 1) // d + 1)
            assert r["softmax_sum"][t, 0] == nvis
            if nvis:
                np.testing.assert_allclose(r["out"][t, 0], vc[:nvis].mean(0), rtol=1e-12, atol=1e-14)


def test_attention_empty_rows():
    c = _small_case(S=100, n1=4, n2=2, l=32, d=16)
    r = _run(c)
    empty = np.arange(31)             # t < l - 1 sees no block
    assert np.all(r["out"][empty] == 0)
    assert np.all(np.isneginf(r["softmax_max"][empty]))
    assert np.all(r["softmax_sum"][empty] == 0)
    assert np.all(r["topk"][empty] == -1)
    assert not np.any(r["topk"][31:, :, 0] == -1)


def test_gqa_equals_mha_with_replicated_kv_heads():
    c = _small_case(S=260, n1=8, n2=2, d1=32, d2=32, count=3)
    r = _run(c)
    G = 4
    c2 = dict(c)
    c2["kc"] = c["kc"].repeat_interleave(G, 1)
    c2["vc"] = c["vc"].repeat_interleave(G, 1)
    r2 = _run(c2)
    np.testing.assert_array_equal(r["out"], r2["out"])
    np.testing.assert_array_equal(r["softmax_max"], r2["softmax_max"])
    np.testing.assert_array_equal(r["softmax_sum"], r2["softmax_sum"])
    # the group score of GQA is the sum of the per-head scores of MHA
    np.testing.assert_allclose(r["score"], r2["score"].reshape(260, 2, G, -1).sum(2),
                               rtol=1e-13, atol=1e-15)


def test_group_score_is_sum_of_head_importances():
    """Step 5 against steps 2+4 recomputed per head from the one-hot readout."""
    c = _small_case(S=180, n1=4, n2=1, d1=16, d2=16, l=32, d=16, lp=32)
    n_cmp = c["kc"].shape[0]
    vc = torch.zeros(n_cmp, 1, 16)
    vc[torch.arange(n_cmp), 0, torch.arange(n_cmp)] = 1.0
    c["vc"] = vc.to(torch.bfloat16)
    r = _run(c)
    n_sel = int(c["cu_sel"][-1])
    for t in [40, 77, 120, 179]:
        nvis = min(n_cmp, (t - 31) // 16 + 1)
        tot = np.zeros(n_sel)
        for h in range(4):
            tot += oracle.importance(r["out"][t, h, :nvis], nvis, 2, 2, n_sel)
        np.testing.assert_allclose(r["score"][t, 0, :n_sel], tot, rtol=1e-13, atol=1e-15)


def test_topk_in_pipeline_matches_torch_topk_on_candidates():
    c = _small_case(S=700, n1=4, n2=2, d1=32, d2=16, l=32, d=16, lp=64, count=5)
    r = _run(c)
    for t in range(31, 700, 7):
        ncand = min(int(c["cu_sel"][-1]), t // 64 + 1)      # j * l' <= t
        for g in range(2):
            assert r["ncand"][t, g] == ncand
            s = torch.from_numpy(r["score"][t, g, :ncand])
            k = min(5, ncand)
            sel = torch.sort(s, descending=True, stable=True).indices[:k]
            assert r["topk"][t, g].tolist() == sorted(sel.tolist()) + [-1] * (5 - k)


def test_short_query_offset_aligns_last_query_to_last_token():
    """Bottom-right alignment reading: the last of S_q queries sits at the
    last raw token covered by the compressed blocks."""
    full = _small_case(S=512, n1=2, n2=1, l=64, d=32, lp=64, count=4)
    rf = _run(full)
    short = dict(full)
    short["q"] = full["q"][-64:]
    short["cu_q"] = np.array([64], dtype=np.int32)
    rs = _run(short)
    np.testing.assert_array_equal(rs["out"], rf["out"][-64:])
    np.testing.assert_array_equal(rs["topk"], rf["topk"][-64:])


def test_varlen_sequences_are_independent():
    seqs = [90, 0, 257, 31, 140]
    c = _small_case(seqs=seqs, n1=4, n2=2, d1=16, d2=16, l=32, d=16, lp=32, count=3)
    r = _run(c)
    starts = np.concatenate([[0], c["cu_q"][:-1]])
    cstarts = np.concatenate([[0], c["cu_cmp"][:-1]])
    for b, S in enumerate(seqs):
        if S == 0:
            continue
        one = dict(c)
        one["q"] = c["q"][starts[b]:starts[b] + S]
        one["kc"] = c["kc"][cstarts[b]:c["cu_cmp"][b]]
        one["vc"] = c["vc"][cstarts[b]:c["cu_cmp"][b]]
        one["cu_q"] = np.array([S], np.int32)
        one["cu_cmp"] = np.array([c["cu_cmp"][b] - cstarts[b]], np.int32)
        one["cu_sel"] = np.array([-(-S // 32)], np.int32)
        if one["kc"].shape[0] == 0:
            one["kc"] = torch.zeros(0, 2, 16, dtype=torch.bfloat16)
            one["vc"] = torch.zeros(0, 2, 16, dtype=torch.bfloat16)
        ro = _run(one)
        np.testing.assert_array_equal(ro["out"], r["out"][starts[b]:starts[b] + S])
        np.testing.assert_array_equal(ro["topk"], r["topk"][starts[b]:starts[b] + S])


def test_row_sample_equals_full_run():
    c = _small_case(S=333, n1=4, n2=2)
    full = _run(c)
    rows = workloads.sample_rows(c["cu_q"], first=20, last=20, every=17)
    part = _run(c, rows=rows)
    np.testing.assert_array_equal(part["out"], full["out"][rows])
    np.testing.assert_array_equal(part["topk"], full["topk"][rows])


def test_tiny_workload_end_to_end_shapes_and_candidates():
    wl = workloads.TINY
    x = wl.generate()
    kc, cuc = oracle.compress(x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=oracle.BF16)
    vc, _ = oracle.compress(x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=oracle.BF16)
    assert kc.shape == (63, 1, 64) and vc.shape == (63, 1, 64)
    r = oracle.compress_attention(x["q"], kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count,
                                  x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    assert r["out"].shape == (1024, 4, 64)
    assert r["topk"].shape == (1024, 1, 8)
    t = np.arange(1024)
    kstar = np.where(t < 31, 0, np.minimum(8, np.minimum(t // 64 + 1, 16)))
    assert np.array_equal((r["topk"][:, 0] >= 0).sum(1), kstar)
    sel = r["topk"][:, 0]
    for row in sel:
        v = row[row >= 0]
        assert np.all(np.diff(v) > 0)
