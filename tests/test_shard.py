"""Sharding one problem by KV-head group (no communication): the balanced
group split, and the shards' work items covering every (query row, KV group)
pair of the problem exactly once.  Host only: the planner runs on the CPU."""
import numpy as np
import pytest

import sparse_long_context_nsa_b200 as nsa
from sparse_long_context_nsa_b200 import _build


@pytest.fixture(scope="module", autouse=True)
def lib():
    _build.build()
    return nsa.load()


@pytest.mark.parametrize("n2", [1, 2, 3, 4, 7, 8, 16])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_group_split_is_balanced_contiguous_partition(n2, world):
    owner = np.full(n2, -1)
    counts = []
    prev_end = 0
    for r in range(world):
        b, c = nsa.nsa_shard_groups(n2, world, r)
        assert b == prev_end, "shards are contiguous and in rank order"
        assert (owner[b:b + c] == -1).all()
        owner[b:b + c] = r
        counts.append(c)
        prev_end = b + c
    assert prev_end == n2 and (owner >= 0).all()
    assert max(counts) - min(counts) <= 1


def test_group_split_rejects_bad_arguments():
    for args in ((0, 1, 0), (4, 0, 0), (4, 2, 2), (4, 2, -1)):
        with pytest.raises(ValueError):
            nsa.nsa_shard_groups(*args)


CASES = [
    # (seqlens, q_last, n1, n2, d1, d2, l, d, lp, count)
    ((1024,), None, 4, 1, 64, 64, 32, 16, 64, 8),
    ((0, 900, 31, 47, 1, 2049, 16, 600), None, 16, 4, 64, 64, 32, 16, 64, 8),
    ((4096, 3000, 2001), 100, 32, 4, 64, 64, 64, 32, 64, 16),
    ((16384,), None, 64, 4, 128, 128, 32, 16, 64, 16),
    ((2500,), None, 64, 8, 256, 256, 32, 16, 64, 8),      # one M-tile per item (D2 > 128)
]


def _prefix(x):
    return np.cumsum(np.asarray(x, dtype=np.int64)).astype(np.int32)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"n2={c[3]}-b{len(c[0])}")
@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_shard_plans_cover_every_row_and_group_once(case, world):
    seqs, q_last, n1, n2, d1, d2, l, d, lp, count = case
    qlen = [min(q_last, s) if q_last else s for s in seqs]
    cuq = _prefix(qlen)
    cuc = nsa.nsa_compress_out_len(_prefix(seqs), l, d)
    cus = _prefix([-(-s // lp) for s in seqs])
    t1 = int(cuq[-1])
    cover = np.zeros((t1, n2), dtype=np.int64)
    total_ws = 0
    for r in range(world):
        b, c = nsa.nsa_shard_groups(n2, world, r)
        items = nsa.nsa_compress_attention_shard_plan(n1, n2, d1, d2, l, d, lp, count, cuq, cuc, cus, b, c)
        for row0, ntok, g in items:
            assert b <= g < b + c, "an item outside the shard's groups"
            assert ntok >= 1
            cover[row0:row0 + ntok, g] += 1
        total_ws += nsa.nsa_compress_attention_shard_workspace_size(n1, n2, d1, d2, l, d, lp, count, cuq, cuc,
                                                                    cus, b, c)
    assert (cover == 1).all(), "shards must partition the (query row, KV group) pairs exactly"
    # items never straddle two sequences
    full = nsa.nsa_compress_attention_shard_plan(n1, n2, d1, d2, l, d, lp, count, cuq, cuc, cus, 0, n2)
    bounds = np.concatenate([[0], cuq])
    for row0, ntok, _ in full:
        b = np.searchsorted(bounds, row0, side="right") - 1
        assert row0 + ntok <= bounds[b + 1]
    assert len(full) == sum(len(nsa.nsa_compress_attention_shard_plan(
        n1, n2, d1, d2, l, d, lp, count, cuq, cuc, cus, *nsa.nsa_shard_groups(n2, world, r))) for r in range(world))


def test_shard_range_is_checked():
    cuq = _prefix([1024])
    cuc = nsa.nsa_compress_out_len(cuq, 32, 16)
    for b, c in ((-1, 1), (0, 3), (2, 1), (1, -1)):
        with pytest.raises(ValueError):
            nsa.nsa_compress_attention_shard_plan(8, 2, 64, 64, 32, 16, 64, 8, cuq, cuc, _prefix([16]), b, c)
