"""Host arithmetic of bench.py checked against brute force: the attended-key
count behind the selection-attention FLOPs, and the visible compressed blocks
behind the compressed-attention FLOPs."""
import numpy as np

import bench
import workloads


def _keys_brute(topk, cu_q, cu_kv, lp):
    out = np.zeros(topk.shape[:2], np.int64)
    q0 = k0 = 0
    for b in range(len(cu_q)):
        sq, skv = int(cu_q[b]) - q0, int(cu_kv[b]) - k0
        for tl in range(sq):
            t = tl + skv - sq
            for g in range(topk.shape[1]):
                keys = set()
                for j in topk[q0 + tl, g]:
                    if j < 0:
                        continue
                    keys.update(p for p in range(j * lp, j * lp + lp) if p <= t and p < skv)
                out[q0 + tl, g] = len(keys)
        q0, k0 = int(cu_q[b]), int(cu_kv[b])
    return out


def test_row_keys_matches_brute_force():
    rng = np.random.default_rng(3)
    lp = 16
    cq = np.cumsum([50, 0, 30, 7]).astype(np.int32)
    ck = np.cumsum([70, 20, 30, 100]).astype(np.int32)
    tk = rng.integers(-1, 8, size=(int(cq[-1]), 2, 5)).astype(np.int32)
    tk[::3, :, 1] = tk[::3, :, 0]                        # repeats count once
    assert np.array_equal(bench.row_keys(tk, cq, ck, lp), _keys_brute(tk, cq, ck, lp))


def test_select_flops_counts_all_heads():
    wl = workloads.TINY
    keys = np.full((10, wl.n2), 64, np.int64)
    assert bench.select_flops(wl, keys) == 2.0 * (wl.d1 + wl.d2) * (wl.n1 // wl.n2) * 640


def test_visible_pairs_matches_brute_force():
    wl = workloads.TINY
    S, l, d = wl.seqlens[0], wl.l, wl.d
    n_cmp = (S - l) // d + 1
    brute = sum(sum(1 for i in range(n_cmp) if i * d + l - 1 <= t) for t in range(S))
    assert bench.visible_pairs(wl) == brute
