"""Head-group shards on the GPU: the outputs of the shards of one problem,
each computed by nsa_compress_attention_shard into the same buffers, are
bitwise those of the whole-problem call, and rows outside a shard are left
untouched."""
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


@pytest.mark.parametrize("seqs,n1,n2,dd,world", [
    ((3000, 700, 0, 1500), 32, 4, 64, 2),
    ((5000,), 64, 8, 128, 3),
    ((2000, 1300), 16, 2, 256, 2),          # one M-tile per item
])
def test_shards_reassemble_the_whole_problem(nsa, seqs, n1, n2, dd, world):
    wl = workloads.Workload("shard", seqs, n1, n2, dd, dd, 32, 16, 64, 8, dd ** -0.5, seed=31)
    x = wl.generate(device="cuda")
    cuc = nsa.nsa_compress_out_len(x["cu_seqlens"], wl.l, wl.d)
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"])
    args = (x["q"], kc, vc, wl.scale, n1, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"])
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(n1, n2, dd, dd, wl.l, wl.d, wl.lp, wl.count,
                                                               x["cu_seqlens_q"], cuc, x["cu_sel_kv"]),
                     dtype=torch.uint8, device="cuda")
    full = nsa.nsa_compress_attention(*args, workspace=ws)
    assert nsa.nsa_workspace_status(ws) == 0
    t1 = x["q"].shape[0]
    G = n1 // n2
    # sentinels: every row must be written by exactly the shard that owns it
    outs = (torch.full((t1, n1, dd), 7.0, dtype=x["q"].dtype, device="cuda"),
            torch.full((t1, n2, wl.count), -7, dtype=torch.int32, device="cuda"),
            torch.full((t1, n1, 8), 7.0, device="cuda"), torch.full((t1, n1, 8), 7.0, device="cuda"))
    for r in range(world):
        b, c = nsa.nsa_shard_groups(n2, world, r)
        before = [o.clone() for o in outs]
        sws = torch.empty(nsa.nsa_compress_attention_shard_workspace_size(
            n1, n2, dd, dd, wl.l, wl.d, wl.lp, wl.count, x["cu_seqlens_q"], cuc, x["cu_sel_kv"], b, c),
            dtype=torch.uint8, device="cuda")
        nsa.nsa_compress_attention_shard(*args, b, c, out=outs, workspace=sws)
        assert nsa.nsa_workspace_status(sws) == 0
        # outside the shard nothing changed
        hs = slice(b * G, (b + c) * G)
        for o, o0, ax_n in ((outs[0], before[0], n1), (outs[2], before[2], n1), (outs[3], before[3], n1)):
            mask = torch.ones(ax_n, dtype=torch.bool, device="cuda")
            mask[hs] = False
            assert torch.equal(o[:, mask], o0[:, mask])
        gmask = torch.ones(n2, dtype=torch.bool, device="cuda")
        gmask[b:b + c] = False
        assert torch.equal(outs[1][:, gmask], before[1][:, gmask])
    assert torch.equal(outs[0].view(torch.int16), full[0].view(torch.int16))
    assert torch.equal(outs[1], full[1])
    assert torch.equal(outs[2], full[2]) and torch.equal(outs[3], full[3])
