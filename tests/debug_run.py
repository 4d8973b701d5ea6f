"""Runs every compute entry point on small seeded inputs and saves the outputs
(torch.save) to the path given: executed twice by tests/test_debug_gpu.py, once
with NSA_DEBUG=1 (the debug library with device bounds checks and guard bands
after the binding's allocations) and once without."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import sparse_long_context_nsa_b200 as nsa  # noqa: E402
import workloads  # noqa: E402


def main(path):
    wl = workloads.Workload("case", (300, 0, 40, 1777), 16, 4, 64, 64, 32, 16, 64, 8, 0.125, "bf16", seed=51)
    x = wl.generate(device="cuda")
    cu, cuq, cus = x["cu_seqlens"], x["cu_seqlens_q"], x["cu_sel_kv"]
    out = {}
    kc, vc = nsa.nsa_compress(x["k"], x["v"], x["w"], wl.l, wl.d, cu)
    assert nsa.nsa_compress_status() == 0
    cuc = nsa.nsa_compress_out_len(cu, wl.l, wl.d)
    att = nsa.nsa_compress_attention(x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus)
    rng = np.random.default_rng(52)
    am = torch.from_numpy(rng.random((1777, 128)) < 0.3).cuda()
    tm = torch.from_numpy(rng.random((1777, 32)) < 0.3).cuda()
    msk = nsa.nsa_compress_attention(x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus,
                                     atten_mask=am, topk_mask=tm)
    sel = nsa.nsa_select_attention(x["q"], x["k"], x["v"], att[1], wl.scale, wl.n1, wl.lp, cuq, cu)
    gout = workloads.grad_output(wl).cuda()
    grads = nsa.nsa_compress_attention_backward(x["q"], kc, vc, att[0], gout, att[2], att[3], wl.scale, wl.n1, wl.l,
                                                wl.d, cuq, cuc)
    cgr = nsa.nsa_compress_backward(x["k"], x["v"], x["w"], grads[1], grads[2], wl.l, wl.d, cu)
    # paged: every sequence's blocks in pages of 16, in order
    ncs = np.diff(np.concatenate([[0], cuc]))
    npg = [-(-int(n) // 16) for n in ncs]
    table = torch.full((len(ncs), max(npg) + 1), -1, dtype=torch.int32)
    kp = torch.zeros(sum(npg), 16, wl.n2, wl.d1, dtype=kc.dtype, device="cuda")
    vp = torch.zeros_like(kp)
    o = 0
    for b, n in enumerate(npg):
        table[b, :n] = torch.arange(o, o + n, dtype=torch.int32)
        o += n
    table = table.cuda()
    nsa.nsa_compress_paged(x["k"], x["v"], x["w"], wl.l, wl.d, cu, kp, vp, table)
    assert nsa.nsa_compress_status() == 0
    pag = nsa.nsa_compress_attention_paged(x["q"], kp, vp, table, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq,
                                           cuc, cus)
    b, c = nsa.nsa_shard_groups(wl.n2, 2, 1)
    shd = nsa.nsa_compress_attention_shard(x["q"], kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq, cuc,
                                           cus, b, c)
    for name, ts in (("compress", (kc, vc)), ("attention", att), ("masked", msk), ("select", sel),
                     ("backward", grads), ("compress_backward", cgr), ("paged", pag), ("shard", shd)):
        out[name] = [t.cpu() if t is not None else None for t in ts]
    torch.cuda.synchronize()
    out["debug_lib_loaded"] = any(nsa.LIB_DEBUG_PATH in line for line in open("/proc/self/maps"))
    torch.save(out, path)


if __name__ == "__main__":
    main(sys.argv[1])
