"""Benchmark of the NSA compressed-attention hot path on B200.

One step = nsa_compress (raw K/V -> block tokens) + nsa_compress_attention
(scores, softmax, PV, importance band, group sum, top-k) over one batch of
seeded synthetic inputs, launched through the C ABI.  The default workload is
the largest single-GPU one: one sequence of 131072 tokens, 128 query heads in
8 KV groups.  The same JSON line also carries the bandwidth-bound compress of
262144 raw tokens (4 sequences of 65536, N2 = 8, D = 128, l = 128, d = 64) and
the short-query attention of its last 128 tokens per sequence, each timed in
the same run with its own roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle as reference arm

Prints one JSON line (rank 0).  `value` is algorithmic compressed-attention
TFLOP/s over the whole step (compress + attention, device time, inputs
resident in HBM), summed over ranks (weak scaling: every rank runs its own
independent batch, no collective on the data path).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = ("compressed-attn TFLOP/s + query tok/s (fwd incl. top-k), % bf16 peak; "
          "compress GB/s")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = os.path.join(ROOT, "sparse_long_context_nsa_b200", "csrc")
# sources whose change invalidates a recorded DRAM-traffic figure
ATTN_SRC = [os.path.join(_CSRC, "nsa_attention.cu")]
CMP_SRC = [os.path.join(_CSRC, "nsa_compress.cu")]
SEL_SRC = [os.path.join(_CSRC, "nsa_select.cu")]
BWD_SRC = [os.path.join(_CSRC, "nsa_backward.cu")]


# ------------------------------------------------------------------ work
def visible_pairs(wl: workloads.Workload) -> int:
    """sum over query rows of the number of visible compressed blocks."""
    tot = 0
    for S, sq in zip(wl.seqlens, wl.q_lengths()):
        n_cmp = 0 if S < wl.l else (S - wl.l) // wl.d + 1
        off = max(0, (n_cmp - 1) * wl.d + wl.l - sq) if n_cmp > 0 else 0
        t = np.arange(sq, dtype=np.int64) + off
        nv = np.where(t < wl.l - 1, 0, np.minimum(n_cmp, (t - wl.l + 1) // wl.d + 1))
        tot += int(nv.sum())
    return tot


def attention_flops(wl) -> float:
    return 2.0 * (wl.d1 + wl.d2) * wl.n1 * visible_pairs(wl)


def backward_flops(wl) -> float:
    """algorithmic FLOPs of the attention backward: the five contractions per
    visible (row, block) pair and head -- S = q k (recomputed), dP = dout v,
    dv += P dout, dq += dS k, dk += dS q -- 2 (3 D1 + 2 D2) each."""
    return 2.0 * (3 * wl.d1 + 2 * wl.d2) * wl.n1 * visible_pairs(wl)


def backward_executed_flops(wl) -> float:
    """tensor FLOPs the kernels issue: the dq pass recomputes S and dP, the
    dk/dv pass recomputes them again."""
    return 2.0 * (4 * wl.d1 + 3 * wl.d2) * wl.n1 * visible_pairs(wl)


def compress_backward_bytes(wl) -> float:
    """bytes the compression backward must move once: raw k, v (storage dtype)
    and w in, dkcmp / dvcmp (fp32) in, dk, dv (fp32) and dw out."""
    tc = sum(0 if S < wl.l else (S - wl.l) // wl.d + 1 for S in wl.seqlens)
    return float(wl.t2 * wl.n2 * (wl.d1 + wl.d2) * (2 + 4) + tc * wl.n2 * (wl.d1 + wl.d2) * 4
                 + wl.l * wl.n2 * (2 + 4))


def compress_bytes(wl) -> float:
    e = 2
    tc = sum(0 if S < wl.l else (S - wl.l) // wl.d + 1 for S in wl.seqlens)
    return float(wl.t2 * wl.n2 * (wl.d1 + wl.d2) * e + tc * wl.n2 * (wl.d1 + wl.d2) * e
                 + wl.l * wl.n2 * e)


def row_keys(topk, cu_q, cu_kv, lp):
    """(T1, N2): keys each (query row, KV group) attends to through its listed
    blocks: block j gives keys j*lp .. j*lp+lp-1 up to the row's key position
    t and the end of the sequence (repeats and -1 give none)."""
    out = np.zeros(topk.shape[:2], np.int64)
    q0 = k0 = 0
    for b in range(len(cu_q)):
        sq, skv = int(cu_q[b]) - q0, int(cu_kv[b]) - k0
        if sq > 0:
            t = (np.arange(sq, dtype=np.int64) + skv - sq)[:, None, None]
            srt = np.sort(topk[q0:q0 + sq].astype(np.int64), axis=-1)
            first = np.ones_like(srt, dtype=bool)
            first[..., 1:] = srt[..., 1:] != srt[..., :-1]
            kk = np.minimum(np.minimum(lp, t - srt * lp + 1), skv - srt * lp)
            out[q0:q0 + sq] = np.where((srt >= 0) & first & (kk > 0), kk, 0).sum(-1)
        q0, k0 = int(cu_q[b]), int(cu_kv[b])
    return out


def select_flops(wl, keys) -> float:
    """algorithmic FLOPs of selection attention: QK^T and PV over the attended keys, all heads."""
    return 2.0 * (wl.d1 + wl.d2) * (wl.n1 // wl.n2) * float(np.sum(keys))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash(paths):
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(kind, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    this workload and the kernel source still matches the one it was taken on."""
    p = os.path.join(ROOT, "profiles", f"{kind}_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = {"attention": ATTN_SRC, "compress": CMP_SRC, "select": SEL_SRC, "backward": BWD_SRC}[kind]
    if d.get("workload") != workload or d.get("source_sha256_16") != src_hash(src):
        return None
    return d.get("bytes_per_launch_full_workload")


# ------------------------------------------------------------ ranks
def rank_workload(name: str, rank: int) -> workloads.Workload:
    """Each rank runs its own independent batch: same shapes, seed offset by rank."""
    wl = workloads.WORKLOADS[name]
    return wl.replace(seed=wl.seed + 1000 * rank)


def max_over_ranks(values, device, world: int):
    """Element-wise max of a list of floats over all ranks (identity for one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device, world: int):
    """Element-wise sum of a list of floats over all ranks (identity for one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return t.tolist()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while running."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons = [], set()
        self.stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join()

    def result(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import sparse_long_context_nsa_b200 as nsa
    from sparse_long_context_nsa_b200 import _build
    if rank == 0:
        _build.build()
    if world > 1:
        torch.distributed.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = rank_workload(args.workload, rank)
    x = wl.generate(device=str(dev))
    q, k, v, w = x["q"], x["k"], x["v"], x["w"]
    cu, cuq, cus = x["cu_seqlens"], x["cu_seqlens_q"], x["cu_sel_kv"]
    cuc = nsa.nsa_compress_out_len(cu, wl.l, wl.d)
    tc = int(cuc[-1])
    t1 = q.shape[0]
    kc = torch.empty(tc, wl.n2, wl.d1, dtype=q.dtype, device=dev)
    vc = torch.empty(tc, wl.n2, wl.d2, dtype=q.dtype, device=dev)
    outs = (torch.empty(t1, wl.n1, wl.d2, dtype=q.dtype, device=dev),
            torch.empty(t1, wl.n2, wl.count, dtype=torch.int32, device=dev),
            torch.empty(t1, wl.n1, 8, dtype=torch.float32, device=dev),
            torch.empty(t1, wl.n1, 8, dtype=torch.float32, device=dev))
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus),
        dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2

    def step():
        nsa.nsa_compress(k, v, w, wl.l, wl.d, cu, kcmp=kc, vcmp=vc)
        nsa.nsa_compress_attention(q, kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq, cuc,
                                   cus, out=outs, workspace=ws)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.nsa_workspace_status(ws) != 0 or nsa.nsa_compress_status() != 0:
        raise RuntimeError("device-side timeout during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_wall = time.perf_counter()
        for i in range(K):
            flush.zero_()                       # L2 flushed between timed steps
            ev[i][0].record()
            nsa.nsa_compress(k, v, w, wl.l, wl.d, cu, kcmp=kc, vcmp=vc)
            ev[i][1].record()
            nsa.nsa_compress_attention(q, kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq,
                                       cuc, cus, out=outs, workspace=ws)
            ev[i][2].record()
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    st_ws = nsa.nsa_workspace_status(ws)
    if st_ws != 0 or nsa.nsa_compress_status() != 0:
        raise RuntimeError("device-side timeout in the timed region")
    t_cmp = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    t_att = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    step_ms = float(np.sum(t_cmp) + np.sum(t_att))    # device time of the K steps
    att_ms = float(np.mean(t_att))
    cmp_ms = float(np.mean(t_cmp))

    # ---------------- end to end: host buffers through the public API ----------------
    e2e = None
    if not args.no_e2e:
        # As a user streams batches: step i's inputs copy in on one stream while
        # step i-1 computes and step i-2's outputs copy out on another (the two
        # directions use separate copy engines).  Two device buffer sets; every
        # step copies all of its inputs in and all of its outputs back.
        hq, hk, hv, hw = (t.cpu().pin_memory() for t in (q, k, v, w))
        ke = max(3, min(K, args.e2e_steps))
        s_cmp = torch.cuda.current_stream(dev)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        din = [tuple(torch.empty_like(t) for t in (q, k, v, w)) for _ in range(2)]
        dcmp = [(torch.empty_like(kc), torch.empty_like(vc)) for _ in range(2)]
        dout = [tuple(torch.empty_like(t) for t in outs) for _ in range(2)]
        hout = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs) for _ in range(2)]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_cmp[b])            # step i-2 has finished reading these inputs
                for h_, d_ in zip((hq, hk, hv, hw), din[b]):
                    d_.copy_(h_, non_blocking=True)
                ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])               # step i-2's outputs have left this buffer set
            dq, dk, dv, dw = din[b]
            nsa.nsa_compress(dk, dv, dw, wl.l, wl.d, cu, kcmp=dcmp[b][0], vcmp=dcmp[b][1])
            nsa.nsa_compress_attention(dq, dcmp[b][0], dcmp[b][1], wl.scale, wl.n1, wl.l, wl.d, wl.lp,
                                       wl.count, cuq, cuc, cus, out=dout[b], workspace=ws)
            ev_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                for h_, d_ in zip(hout[b], dout[b]):
                    h_.copy_(d_, non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_cmp)
        s_in.wait_stream(s_cmp)
        for i in range(ke):
            e2e_step(i)
        s_cmp.wait_stream(s_in)
        s_cmp.wait_stream(s_out)
        e1.record(s_cmp)
        torch.cuda.synchronize()
        if nsa.nsa_workspace_status(ws) != 0 or nsa.nsa_compress_status() != 0:
            raise RuntimeError("device-side timeout in the end-to-end steps")
        # the overlapped steps computed what the resident steps did (both are deterministic)
        last = hout[(ke - 1) % 2]
        if not (torch.equal(last[1], outs[1].cpu()) and torch.equal(last[0][:64], outs[0][:64].cpu())):
            raise RuntimeError("end-to-end outputs differ from the resident run")
        e2e_ms = e0.elapsed_time(e1) / ke
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hw))
        d2h = sum(t.numel() * t.element_size() for t in hout[0])
        e2e = {"ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": ke, "overlap": "copy-in, compute and copy-out of consecutive steps on three streams"}

    # ---------- the optional masks of steps 1 and 6 (seeded, 30 % set) ----------
    msk = None
    if not args.no_masks:
        rng = np.random.default_rng(wl.seed + 77)
        sq = np.diff(np.concatenate([[0], cuq]))
        ncs = np.diff(np.concatenate([[0], cuc]))
        nss = np.diff(np.concatenate([[0], cus]))
        am = rng.random((int(sq.max()), max(1, int(ncs.max())))) < 0.3
        tm = rng.random((int(sq.max()), max(1, int(nss.max())))) < 0.3
        am_d, tm_d = torch.from_numpy(am).to(dev), torch.from_numpy(tm).to(dev)
        mouts = tuple(torch.empty_like(t) for t in outs)

        mws = torch.empty(nsa.nsa_compress_attention_masked_workspace_size(
            wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus), dtype=torch.uint8, device=dev)

        def masked_call():
            nsa.nsa_compress_attention(q, kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus,
                                       out=mouts, workspace=mws, atten_mask=am_d, topk_mask=tm_d)

        for _ in range(max(args.warmup, 0)):
            flush.zero_()
            masked_call()
        km = max(3, min(K, args.select_steps))
        mev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(km)]
        for i in range(km):
            flush.zero_()
            mev[i][0].record()
            masked_call()
            mev[i][1].record()
        torch.cuda.synchronize()
        if nsa.nsa_workspace_status(mws) != 0:
            raise RuntimeError("device-side timeout in masked attention")
        # attended (row, block) pairs: visible by the causal rule and not masked
        pairs = 0
        for b in range(len(cuq)):
            n_q, n_c = int(sq[b]), int(ncs[b])
            if n_q == 0 or n_c == 0:
                continue
            off = max(0, (n_c - 1) * wl.d + wl.l - n_q)
            tpos = np.arange(n_q)[:, None] + off
            vis = np.arange(n_c)[None, :] * wl.d + wl.l - 1 <= tpos
            pairs += int((vis & ~am[:n_q, :n_c]).sum())
        msk = dict(ms=float(np.mean([e[0].elapsed_time(e[1]) for e in mev])), steps=km,
                   flops=2.0 * (wl.d1 + wl.d2) * wl.n1 * pairs, am=am, tm=tm)

    # ---------- selection attention over the step's own top-k lists ----------
    sel = None
    if not args.no_select:
        topk = outs[1]
        sws = torch.empty(nsa.nsa_select_attention_workspace_size(wl.n1, wl.n2, wl.d1, wl.d2, wl.lp, wl.count,
                                                                  cuq, cu), dtype=torch.uint8, device=dev)
        sout = (torch.empty(t1, wl.n1, wl.d2, dtype=q.dtype, device=dev),
                torch.empty(t1, wl.n1, dtype=torch.float32, device=dev))

        def sel_call():
            nsa.nsa_select_attention(q, k, v, topk, wl.scale, wl.n1, wl.lp, cuq, cu, out=sout, workspace=sws)

        for _ in range(max(args.warmup, 0)):
            flush.zero_()
            sel_call()
        torch.cuda.synchronize()
        ks = max(3, min(K, args.select_steps))
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(ks)]
        for i in range(ks):
            flush.zero_()
            sev[i][0].record()
            sel_call()
            sev[i][1].record()
        torch.cuda.synchronize()
        if nsa.nsa_workspace_status(sws) != 0:
            raise RuntimeError("device-side timeout in selection attention")
        tk_host = topk.cpu().numpy()
        sel = dict(ms=float(np.mean([e[0].elapsed_time(e[1]) for e in sev])), steps=ks,
                   keys=row_keys(tk_host, cuq, cu, wl.lp), topk=tk_host)

    # ---------- backward: gradients of the step's attention and compression ----------
    bwd = None
    if not args.no_backward:
        gout = workloads.grad_output(wl, device=str(dev))
        att, _, smax, ssum = outs
        bws = torch.empty(nsa.nsa_compress_attention_backward_workspace_size(
            wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, cuq, cuc), dtype=torch.uint8, device=dev)
        grads = (torch.empty(t1, wl.n1, wl.d1, dtype=torch.float32, device=dev),
                 torch.empty(tc, wl.n2, wl.d1, dtype=torch.float32, device=dev),
                 torch.empty(tc, wl.n2, wl.d2, dtype=torch.float32, device=dev))
        cws = torch.empty(nsa.nsa_compress_backward_workspace_size(cu, wl.l, wl.d), dtype=torch.uint8, device=dev)
        cgrads = (torch.empty(k.shape, dtype=torch.float32, device=dev),
                  torch.empty(v.shape, dtype=torch.float32, device=dev),
                  torch.empty(wl.l, wl.n2, dtype=torch.float32, device=dev))

        def bwd_att():
            nsa.nsa_compress_attention_backward(q, kc, vc, att, gout, smax, ssum, wl.scale, wl.n1, wl.l, wl.d,
                                                cuq, cuc, grads=grads, workspace=bws)

        def bwd_cmp():
            nsa.nsa_compress_backward(k, v, w, grads[1], grads[2], wl.l, wl.d, cu, grads=cgrads, workspace=cws)

        for _ in range(max(args.warmup, 0)):
            flush.zero_()
            bwd_att()
            bwd_cmp()
        kb = max(3, min(K, args.backward_steps))
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(kb)]
        for i in range(kb):
            flush.zero_()
            bev[i][0].record()
            bwd_att()
            bev[i][1].record()
            bwd_cmp()
            bev[i][2].record()
        torch.cuda.synchronize()
        if nsa.nsa_workspace_status(bws) != 0 or nsa.nsa_workspace_status(cws) != 0:
            raise RuntimeError("device-side timeout in the backward")
        bwd = dict(att_ms=float(np.mean([e[0].elapsed_time(e[1]) for e in bev])),
                   cmp_ms=float(np.mean([e[1].elapsed_time(e[2]) for e in bev])), steps=kb,
                   launches=(5 if wl.d2 > 128 else 4) + 2 + (len(wl.seqlens) - 1) // 96,
                   gsample=gout[:min(int(wl.seqlens[0]), 16384), :wl.n1 // wl.n2].cpu())
        del grads, cgrads, bws, gout

    dec = None
    if not args.no_decode:
        dec = time_decode(args, nsa, dev, rank, flush)

    side = None
    if not args.no_side:
        del flush
        side = time_side_case(args, nsa, dev, rank)

    return dict(wl=wl, K=K, step_ms=step_ms, att_ms=att_ms, cmp_ms=cmp_ms, t1=t1, wall=t_wall,
                clocks=clk.result(), e2e=e2e, sel=sel, msk=msk, side=side, x=x, bwd=bwd, dec=dec,
                launches_per_step=1 + 1 + (len(wl.seqlens) - 1) // 96)


def decode_bytes(dw) -> float:
    """bytes a decode step must move: every sequence's compressed K/V once, plus
    q, attention_out, the statistics and the top-k lists."""
    e = 2
    kv = dw.batch * dw.n_cmp * dw.n2 * (dw.d1 + dw.d2) * e
    io = dw.batch * dw.n1 * (dw.d1 + dw.d2) * e + dw.batch * dw.n1 * 16 * 4 + dw.batch * dw.n2 * dw.count * 4
    return float(kv + io)


def time_decode(args, nsa, dev, rank, flush):
    """One decode step over a paged compressed cache (one query per sequence),
    L2 flushed before every call."""
    dw = workloads.DECODE_64x64K
    dw = dataclasses.replace(dw, seed=dw.seed + rank)
    x = dw.generate(device=str(dev))
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        dw.n1, dw.n2, dw.d1, dw.d2, dw.l, dw.d, dw.lp, dw.count, x["cu_seqlens_q"], x["cu_cmp_kv"], x["cu_sel_kv"]),
        dtype=torch.uint8, device=dev)

    def call():
        return nsa.nsa_compress_attention_paged(x["q"], x["kcmp_pages"], x["vcmp_pages"], x["block_table"], dw.scale,
                                                dw.n1, dw.l, dw.d, dw.lp, dw.count, x["cu_seqlens_q"],
                                                x["cu_cmp_kv"], x["cu_sel_kv"], workspace=ws)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        call()
    n = max(3, min(args.steps, args.decode_steps))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for i in range(n):
        flush.zero_()
        evs[i][0].record()
        res = call()
        evs[i][1].record()
    torch.cuda.synchronize()
    if nsa.nsa_workspace_status(ws) != 0:
        raise RuntimeError("device-side timeout in paged decode")
    return dict(wl=dw, ms=float(np.mean([e[0].elapsed_time(e[1]) for e in evs])), steps=n, x=x, res=res)


def decode_cpu_baseline(dw, x, nseq=16):
    """The oracle as it stands on the first nseq sequences of the decode step
    (their pages gathered into contiguous compressed tensors on the host)."""
    import oracle
    bt = x["block_table"].cpu().numpy()
    kp, vp = x["kcmp_pages"].cpu(), x["vcmp_pages"].cpu()
    kc = torch.cat([kp[bt[b]].reshape(-1, dw.n2, dw.d1)[:dw.n_cmp] for b in range(nseq)])
    vc = torch.cat([vp[bt[b]].reshape(-1, dw.n2, dw.d2)[:dw.n_cmp] for b in range(nseq)])
    q = x["q"][:nseq].cpu()
    t = time.perf_counter()
    oracle.compress_attention(q, kc, vc, dw.scale, dw.l, dw.d, dw.lp, dw.count, x["cu_seqlens_q"][:nseq],
                              x["cu_cmp_kv"][:nseq], x["cu_sel_kv"][:nseq])
    sec = time.perf_counter() - t
    return {"value": nseq / sec, "unit": "decode tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{nseq} of {dw.batch} sequences, all heads, {sec:.2f} s"}


def time_side_case(args, nsa, dev, rank):
    """The bandwidth-bound compress of 262144 raw tokens (4 x 65536, N2 = 8,
    D = 128, l = 128, d = 64) and the compressed attention of the last 128
    queries of each sequence against all of its blocks (N1 = 64, l' = 128,
    count = 32): each timed on its own, L2 flushed before every launch."""
    wl = rank_workload(args.side_workload, rank)
    x = wl.generate(device=str(dev))
    q, k, v, w = x["q"], x["k"], x["v"], x["w"]
    cu, cuq, cus = x["cu_seqlens"], x["cu_seqlens_q"], x["cu_sel_kv"]
    cuc = nsa.nsa_compress_out_len(cu, wl.l, wl.d)
    tc, t1 = int(cuc[-1]), q.shape[0]
    kc = torch.empty(tc, wl.n2, wl.d1, dtype=q.dtype, device=dev)
    vc = torch.empty(tc, wl.n2, wl.d2, dtype=q.dtype, device=dev)
    outs = (torch.empty(t1, wl.n1, wl.d2, dtype=q.dtype, device=dev),
            torch.empty(t1, wl.n2, wl.count, dtype=torch.int32, device=dev),
            torch.empty(t1, wl.n1, 8, dtype=torch.float32, device=dev),
            torch.empty(t1, wl.n1, 8, dtype=torch.float32, device=dev))
    ws = torch.empty(nsa.nsa_compress_attention_workspace_size(
        wl.n1, wl.n2, wl.d1, wl.d2, wl.l, wl.d, wl.lp, wl.count, cuq, cuc, cus), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def timed(fn, n):
        for _ in range(max(args.warmup, 0)):
            flush.zero_()
            fn()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for i in range(n):
            flush.zero_()
            evs[i][0].record()
            fn()
            evs[i][1].record()
        torch.cuda.synchronize()
        return float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))

    n = max(3, min(args.steps, args.side_steps))
    cmp_ms = timed(lambda: nsa.nsa_compress(k, v, w, wl.l, wl.d, cu, kcmp=kc, vcmp=vc), n)
    if nsa.nsa_compress_status() != 0:
        raise RuntimeError("device-side timeout in the 262144-token compress")
    att_ms = timed(lambda: nsa.nsa_compress_attention(q, kc, vc, wl.scale, wl.n1, wl.l, wl.d, wl.lp, wl.count,
                                                      cuq, cuc, cus, out=outs, workspace=ws), n)
    if nsa.nsa_workspace_status(ws) != 0:
        raise RuntimeError("device-side timeout in the short-query attention")
    return dict(wl=wl, cmp_ms=cmp_ms, att_ms=att_ms, steps=n, x={kk: x[kk] for kk in ("k", "v", "w")},
                cu=cu)


def compress_cpu_baseline(wl, x, budget_rows=8192):
    """The oracle's compression as it stands, on the first raw rows of the
    first sequence of a workload (x: generated inputs on any device)."""
    import oracle
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    S0 = min(wl.seqlens[0], budget_rows)
    k, v, w = x["k"][:S0].cpu(), x["v"][:S0].cpu(), x["w"].cpu()
    t0 = time.perf_counter()
    oracle.compress(k, w, wl.l, wl.d, [S0], dtype=dt)
    oracle.compress(v, w, wl.l, wl.d, [S0], dtype=dt)
    dt_s = time.perf_counter() - t0
    nc = 0 if S0 < wl.l else (S0 - wl.l) // wl.d + 1
    nbytes = (S0 + nc) * wl.n2 * (wl.d1 + wl.d2) * 2 + wl.l * wl.n2 * 2
    return {"value": nbytes / dt_s / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {S0} raw rows of K and V of the first sequence, {dt_s:.2f} s"}


def gen_device():
    """Where seeded inputs are drawn: the CUDA generator when a GPU is present
    (the large workloads hold several GB of float32 draws), else the CPU."""
    return "cuda" if torch.cuda.is_available() else "cpu"


def host_inputs(x, rows=None):
    """CPU copies of the generated inputs the oracle needs: k, v, w whole and
    q whole or only the query rows in ``rows``."""
    out = {kk: x[kk] for kk in ("cu_seqlens", "cu_seqlens_q", "cu_sel_kv")}
    for kk in ("k", "v", "w"):
        out[kk] = x[kk].cpu()
    if rows is None:
        out["q"] = x["q"].cpu()
    else:
        idx = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=x["q"].device)
        out["q"] = x["q"].index_select(0, idx).cpu()
    return out


def cpu_baseline(wl, x, budget_s=20.0):
    """The fp64 oracle as it stands, timed on a bounded sample of the workload
    (x: the generated inputs, on any device; the oracle gets CPU copies)."""
    import oracle
    x = {kk: (vv.cpu() if torch.is_tensor(vv) and kk != "q" else vv) for kk, vv in x.items()}
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    # compress: a slice of the raw rows of the first sequence
    S0 = min(wl.seqlens[0], 8192)
    t0 = time.perf_counter()
    oracle.compress(x["k"][:S0], x["w"], wl.l, wl.d, [S0], dtype=dt)
    oracle.compress(x["v"][:S0], x["w"], wl.l, wl.d, [S0], dtype=dt)
    t_cmp = time.perf_counter() - t0
    kc, cuc = oracle.compress(x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    # attention: every `stride`-th query row, stride chosen for ~budget_s of CPU
    cq = x["cu_seqlens_q"]
    T1 = int(cq[-1])
    full_pairs = visible_pairs(wl)
    # the cost of a row grows with its position: probe rows spread over the
    # whole query range so that the estimate is the mean cost per row
    probe = np.unique(np.linspace(0, T1 - 1, num=min(T1, 48)).astype(np.int64))
    qp = x["q"].index_select(0, torch.as_tensor(probe, device=x["q"].device)).cpu()
    tp = time.perf_counter()
    oracle.compress_attention(qp, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, cq, cuc,
                              x["cu_sel_kv"], rows=probe, q_rows_only=True)
    per_row = (time.perf_counter() - tp) / probe.size
    nrows = int(max(16, min(T1, budget_s / max(per_row, 1e-6))))
    stride = max(1, T1 // nrows)
    rows = np.arange(0, T1, stride, dtype=np.int64)
    qr = x["q"].index_select(0, torch.as_tensor(rows, device=x["q"].device)).cpu()
    t0 = time.perf_counter()
    oracle.compress_attention(qr, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, cq, cuc,
                              x["cu_sel_kv"], rows=rows, q_rows_only=True)
    t_att = time.perf_counter() - t0
    # visible pairs of the sampled rows (all heads)
    pairs = 0
    prev = 0
    for b, end in enumerate(cq.tolist()):
        sel = rows[(rows >= prev) & (rows < end)]
        S = wl.seqlens[b]
        n_cmp = 0 if S < wl.l else (S - wl.l) // wl.d + 1
        off = max(0, (n_cmp - 1) * wl.d + wl.l - (end - prev)) if n_cmp else 0
        t = sel - prev + off
        pairs += int(np.where(t < wl.l - 1, 0, np.minimum(n_cmp, (t - wl.l + 1) // wl.d + 1)).sum())
        prev = end
    flops = 2.0 * (wl.d1 + wl.d2) * wl.n1 * pairs
    tflops = flops / t_att / 1e12
    cmp_bytes = S0 * wl.n2 * (wl.d1 + wl.d2) * 2 * 2
    return {"value": tflops, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"attention: {rows.size} of {T1} query rows (every {stride}th), all heads, "
                      f"{t_att:.1f} s; compress: first {S0} raw rows of K and V, {t_cmp:.2f} s",
            "compress_gbs": cmp_bytes / t_cmp / 1e9, "seconds": t_att + t_cmp,
            "full_attention_pairs": full_pairs}


def select_cpu_baseline(wl, x, topk, keys, budget_s=8.0):
    """The selection-attention oracle as it stands, on evenly spaced query rows
    (all heads) of the same workload and the same top-k lists."""
    import oracle
    k, v = x["k"].cpu().float(), x["v"].cpu().float()
    cq, ck = x["cu_seqlens_q"], x["cu_seqlens"]
    T1 = int(cq[-1])

    def qrows(r):
        return x["q"].index_select(0, torch.as_tensor(r, device=x["q"].device)).cpu().float()

    probe = np.unique(np.linspace(0, T1 - 1, num=min(T1, 32)).astype(np.int64))
    qp = qrows(probe)
    tp = time.perf_counter()
    oracle.select_attention(qp, k, v, topk, wl.scale, wl.lp, wl.count, cq, ck, rows=probe, q_rows_only=True)
    per_row = (time.perf_counter() - tp) / probe.size
    nrows = int(max(16, min(T1, budget_s / max(per_row, 1e-6))))
    rows = np.unique(np.linspace(0, T1 - 1, num=nrows).astype(np.int64))
    qr = qrows(rows)
    t0 = time.perf_counter()
    oracle.select_attention(qr, k, v, topk, wl.scale, wl.lp, wl.count, cq, ck, rows=rows, q_rows_only=True)
    dt = time.perf_counter() - t0
    return {"value": select_flops(wl, keys[rows]) / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{rows.size} of {T1} evenly spaced query rows, all heads, {dt:.1f} s"}


def masked_cpu_baseline(wl, x, am, tm, budget_s=8.0):
    """The oracle with the same masks, as it stands, on evenly spaced query rows
    (all heads); FLOPs over the attended (visible, unmasked) pairs of those rows."""
    import oracle
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"].cpu(), x["w"].cpu(), wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    cq = x["cu_seqlens_q"]
    T1 = int(cq[-1])

    def run(rows, qr):
        oracle.compress_attention(qr, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, cq, cuc,
                                  x["cu_sel_kv"], rows=rows, q_rows_only=True, atten_mask=am, topk_mask=tm)

    def qrows(r):
        return x["q"].index_select(0, torch.as_tensor(r, device=x["q"].device)).cpu()

    probe = np.unique(np.linspace(0, T1 - 1, num=min(T1, 32)).astype(np.int64))
    qp = qrows(probe)
    tp = time.perf_counter()
    run(probe, qp)
    per_row = (time.perf_counter() - tp) / probe.size
    rows = np.unique(np.linspace(0, T1 - 1, num=int(max(16, min(T1, budget_s / max(per_row, 1e-6))))).astype(np.int64))
    qr = qrows(rows)
    t0 = time.perf_counter()
    run(rows, qr)
    dt_s = time.perf_counter() - t0
    pairs, prev = 0, 0
    for b, end in enumerate(cq.tolist()):
        sel = rows[(rows >= prev) & (rows < end)]
        S = wl.seqlens[b]
        n_cmp = 0 if S < wl.l else (S - wl.l) // wl.d + 1
        if n_cmp and sel.size:
            off = max(0, (n_cmp - 1) * wl.d + wl.l - (end - prev))
            tloc = sel - prev
            vis = np.arange(n_cmp)[None, :] * wl.d + wl.l - 1 <= (tloc + off)[:, None]
            pairs += int((vis & ~am[tloc, :n_cmp]).sum())
        prev = end
    return {"value": 2.0 * (wl.d1 + wl.d2) * wl.n1 * pairs / dt_s / 1e12, "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows.size} of {T1} evenly spaced query rows, all heads, same masks, {dt_s:.1f} s"}


def backward_cpu_baseline(wl, x, gsample, budget_s=10.0):
    """The backward oracle as it stands on a bounded sample: KV group 0 of the
    first sequence's leading S' tokens (S' doubled from 1024 until one call
    takes a quarter of the budget), with its kcmp / vcmp from the oracle's
    compression.  Throughput over the sample's algorithmic FLOPs.  gsample:
    the incoming gradient of those rows and heads (the GPU run's own)."""
    import oracle
    G = wl.n1 // wl.n2
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    s0 = min(int(wl.seqlens[0]), gsample.shape[0])
    if wl.q_last is not None:
        return None
    q0 = x["q"][:s0, :G].cpu()
    k0, v0, w0 = x["k"][:s0, :1].cpu(), x["v"][:s0, :1].cpu(), x["w"][:, :1].cpu()
    gout = gsample
    S = min(1024, s0)
    best = None
    while True:
        cu = np.array([S], dtype=np.int32)
        kc, cuc = oracle.compress(k0[:S], w0, wl.l, wl.d, cu, dtype=dt)
        vc, _ = oracle.compress(v0[:S], w0, wl.l, wl.d, cu, dtype=dt)
        t = time.perf_counter()
        oracle.compress_attention_backward(q0[:S], kc, vc, gout[:S], wl.scale, wl.l, wl.d, cu, cuc)
        dt_s = time.perf_counter() - t
        sw = wl.replace(seqlens=(S,), n1=G, n2=1, q_last=None)
        best = (S, dt_s, backward_flops(sw))
        if dt_s >= budget_s / 4 or S >= s0:
            break
        S = min(2 * S, s0)
    S, dt_s, fl = best
    return {"value": fl / dt_s / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"KV group 0 ({G} heads) of the first {S} tokens of sequence 0: attention backward in "
                      f"fp64, {dt_s:.2f} s"}


def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle (the pages publish no code to run)."""
    if rank != 0:
        return
    import oracle
    wl = workloads.WORKLOADS[args.workload]
    cq = wl.cu_seqlens_q()
    T1 = int(cq[-1])
    rows = np.linspace(0, T1 - 1, num=min(T1, args.ref_rows), dtype=np.int64)
    # inputs drawn where they are cheapest; the oracle gets CPU copies of k, v,
    # w and of the sampled query rows
    x = host_inputs(wl.generate(device=gen_device()), rows)
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.FP16
    kc, cuc = oracle.compress(x["k"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    vc, _ = oracle.compress(x["v"], x["w"], wl.l, wl.d, x["cu_seqlens"], dtype=dt)
    qs = x["q"]

    def step():
        oracle.compress_attention(qs, kc, vc, wl.scale, wl.l, wl.d, wl.lp, wl.count, cq, cuc,
                                  x["cu_sel_kv"], rows=rows, q_rows_only=True)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt_s = (time.perf_counter() - t0) / args.steps
    # algorithmic FLOPs of the sampled rows
    S = wl.seqlens
    pairs, prev = 0, 0
    for b, end in enumerate(cq.tolist()):
        sel = rows[(rows >= prev) & (rows < end)]
        n_cmp = 0 if S[b] < wl.l else (S[b] - wl.l) // wl.d + 1
        off = max(0, (n_cmp - 1) * wl.d + wl.l - (end - prev)) if n_cmp else 0
        t = sel - prev + off
        pairs += int(np.where(t < wl.l - 1, 0, np.minimum(n_cmp, (t - wl.l + 1) // wl.d + 1)).sum())
        prev = end
    flops = 2.0 * (wl.d1 + wl.d2) * wl.n1 * pairs
    val = flops / dt_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": wl.name, "sampled_rows": int(rows.size)},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"{rows.size} evenly spaced query rows of {T1}, all heads, "
                                       "compressed K/V precomputed"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=workloads.LONG_128K.name, choices=list(workloads.WORKLOADS))
    ap.add_argument("--side-workload", default=workloads.SHORTQ_4x64K.name, choices=list(workloads.WORKLOADS),
                    help="workload of the separately timed compress and short-query attention")
    ap.add_argument("--no-side", action="store_true", help="skip the separately timed compress case")
    ap.add_argument("--side-steps", type=int, default=50)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--ref-rows", type=int, default=96)
    ap.add_argument("--no-select", action="store_true", help="skip the selection-attention measurement")
    ap.add_argument("--no-masks", action="store_true", help="skip the masked-attention measurement")
    ap.add_argument("--select-steps", type=int, default=20)
    ap.add_argument("--select-cpu-budget", type=float, default=8.0)
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-decode", action="store_true", help="skip the paged decode measurement")
    ap.add_argument("--decode-steps", type=int, default=20)
    ap.add_argument("--backward-steps", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    r = run_ours(args, rank, world, local_rank)
    wl = r["wl"]
    # max over ranks of the device time of the timed steps
    step_total_ms, att_ms, cmp_ms = max_over_ranks([r["step_ms"], r["att_ms"], r["cmp_ms"]],
                                                   torch.device("cuda", local_rank), world)
    K = r["K"]
    ms_per_step = step_total_ms / K
    flops = attention_flops(wl)
    cbytes = compress_bytes(wl)
    peaks, peak_src = load_peaks()
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    att_tflops = flops / (att_ms * 1e-3) / 1e12
    cmp_gbs = cbytes / (cmp_ms * 1e-3) / 1e9
    e2e = None
    if r["e2e"] is not None:
        e2e_ms = max_over_ranks([r["e2e"]["ms_per_step"]], torch.device("cuda", local_rank), world)[0]
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
               "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"],
               "ms_per_step": e2e_ms, "overlap": r["e2e"]["overlap"]}
    # the separately timed compress / short-query case: max over ranks too
    side_cmp_ms = side_att_ms = None
    if r["side"] is not None:
        side_cmp_ms, side_att_ms = max_over_ranks([r["side"]["cmp_ms"], r["side"]["att_ms"]],
                                                  torch.device("cuda", local_rank), world)
    # selection attention: every rank times its own batch; max of the times,
    # sum of the algorithmic work (the lists differ from rank to rank)
    sel_ms = sel_flops_all = None
    if r["sel"] is not None:
        dev0 = torch.device("cuda", local_rank)
        sel_ms = max_over_ranks([r["sel"]["ms"]], dev0, world)[0]
        sel_flops_all = sum_over_ranks([select_flops(wl, r["sel"]["keys"])], dev0, world)[0]
    dec_ms = None
    if r["dec"] is not None:
        dec_ms = max_over_ranks([r["dec"]["ms"]], torch.device("cuda", local_rank), world)[0]
    bwd_att_ms = bwd_cmp_ms = None
    if r["bwd"] is not None:
        bwd_att_ms, bwd_cmp_ms = max_over_ranks([r["bwd"]["att_ms"], r["bwd"]["cmp_ms"]],
                                                torch.device("cuda", local_rank), world)
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(wl, r["x"], budget_s=args.cpu_budget)
        peak_t = peaks["bf16_tflops"]
        traffic = profile_traffic("attention", wl.name)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.dtype == "bf16" else "fp16", "data": "synthetic",
            "config": {"workload": wl.name, "seqlens": list(wl.seqlens)[:8], "n1": wl.n1, "n2": wl.n2,
                       "d1": wl.d1, "d2": wl.d2, "l": wl.l, "d": wl.d, "lp": wl.lp, "count": wl.count,
                       "l2": "flushed (256 MB write) before every timed step",
                       "parallelism": f"independent batch per GPU x{world}"},
            "query_tok_s": world * r["t1"] / (ms_per_step * 1e-3),
            "attention_kernel": {"ms": att_ms, "tflops": att_tflops,
                                 "pct_of_bf16_peak": 100.0 * att_tflops / peak_t,
                                 "query_tok_s": r["t1"] / (att_ms * 1e-3)},
            "compress_in_step": {"ms": cmp_ms, "gbs": cmp_gbs,
                                 "pct_of_hbm": 100.0 * cmp_gbs / peaks["hbm_gbs"],
                                 "bytes": cbytes, "workload": wl.name},
            "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": att_tflops / peak_t, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "frac_of_sustained": att_tflops / peaks.get("bf16_tflops_sustained", peak_t),
                         "flops_per_launch": flops},
            "clocks": r["clocks"],
            "e2e": e2e,
            "gpu_launches": r["launches_per_step"] * K,
            "cpu_baseline": cpu,
            "wall_s_timed_region": r["wall"],
        }
        if r["side"] is not None:
            swl = r["side"]["wl"]
            sb = compress_bytes(swl)
            sg = sb / (side_cmp_ms * 1e-3) / 1e9
            line["compress_kernel"] = {
                "what": f"nsa_compress alone on {swl.t2} raw tokens ({len(swl.seqlens)} x {swl.seqlens[0]}), "
                        f"N2={swl.n2}, D={swl.d1}, l={swl.l}, d={swl.d}; L2 flushed before every launch",
                "workload": swl.name, "ms": side_cmp_ms, "gbs": sg, "pct_of_hbm": 100.0 * sg / peaks["hbm_gbs"],
                "bytes": sb, "steps": r["side"]["steps"], "gpu_launches": r["side"]["steps"]}
            line["roofline_compress"] = {
                "bound": "hbm", "achieved": sg, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": sg / peaks["hbm_gbs"], "traffic": profile_traffic("compress", swl.name),
                "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": sb}
            sf4 = attention_flops(swl)
            st4 = sf4 / (side_att_ms * 1e-3) / 1e12
            line["shortq_attention"] = {
                "what": f"nsa_compress_attention for the last {swl.q_last} queries of each sequence of the "
                        f"same workload (N1={swl.n1}, l'={swl.lp}, count={swl.count}); L2 flushed before every launch",
                "ms": side_att_ms, "tflops": st4, "pct_of_bf16_peak": 100.0 * st4 / peak_t,
                "query_tok_s": sum(swl.q_lengths()) / (side_att_ms * 1e-3), "flops_per_launch": sf4,
                "steps": r["side"]["steps"], "gpu_launches": r["side"]["steps"],
                "roofline": {"bound": "tensor", "achieved": st4, "peak": peak_t, "unit": "TFLOP/s",
                             "frac": st4 / peak_t, "traffic": None,
                             "peak_source": f"{peak_src} bf16_tflops (burst)"}}
            if not args.no_cpu_baseline and world == 1:
                line["compress_kernel"]["cpu_baseline"] = compress_cpu_baseline(swl, r["side"]["x"])
        if r["msk"] is not None:
            mt = r["msk"]["flops"] / (r["msk"]["ms"] * 1e-3) / 1e12
            line["masked_attention"] = {
                "what": "nsa_compress_attention with atten_mask and topk_mask (seeded, 30 % of entries set); "
                        "FLOPs over the attended (visible, unmasked) pairs",
                "ms": r["msk"]["ms"], "steps": r["msk"]["steps"], "tflops": mt,
                "pct_of_bf16_peak": 100.0 * mt / peak_t, "flops_per_launch": r["msk"]["flops"],
                "unmasked_ms": att_ms, "gpu_launches": r["msk"]["steps"],
                "roofline": {"bound": "tensor", "achieved": mt, "peak": peak_t, "unit": "TFLOP/s",
                             "frac": mt / peak_t, "traffic": None,
                             "peak_source": f"{peak_src} bf16_tflops (burst)"},
                "cpu_baseline": (masked_cpu_baseline(wl, r["x"], r["msk"]["am"], r["msk"]["tm"],
                                                     budget_s=args.select_cpu_budget)
                                 if (not args.no_cpu_baseline and world == 1) else None)}
        if r["sel"] is not None:
            sf = select_flops(wl, r["sel"]["keys"])
            st = sf / (r["sel"]["ms"] * 1e-3) / 1e12                  # this GPU (rank 0)
            line["select_attention"] = {
                "what": "nsa_select_attention over the step's own top-k lists (plan + attention kernels)",
                "ms": sel_ms, "steps": r["sel"]["steps"], "tflops": st,
                "tflops_all_ranks": sel_flops_all / (sel_ms * 1e-3) / 1e12,
                "flops_per_launch": sf,
                "keys_per_row_group": float(np.mean(r["sel"]["keys"])),
                "l2": "flushed (256 MB write) before every timed call",
                "roofline": {"bound": "tensor", "achieved": st, "peak": peak_t, "unit": "TFLOP/s",
                             "frac": st / peak_t, "traffic": profile_traffic("select", wl.name),
                             "peak_source": f"{peak_src} bf16_tflops (burst)"},
                "cpu_baseline": (select_cpu_baseline(wl, r["x"], r["sel"]["topk"], r["sel"]["keys"],
                                                     budget_s=args.select_cpu_budget)
                                 if (not args.no_cpu_baseline and world == 1) else None),
                "gpu_launches": 2 * r["sel"]["steps"],
            }
        if r["bwd"] is not None:
            bf, bx = backward_flops(wl), backward_executed_flops(wl)
            bt = bf / (bwd_att_ms * 1e-3) / 1e12
            cb = compress_backward_bytes(wl)
            cg = cb / (bwd_cmp_ms * 1e-3) / 1e9
            line["backward"] = {
                "what": "nsa_compress_attention_backward (dq, dkcmp, dvcmp from the step's output and "
                        "statistics) then nsa_compress_backward (dk, dv, dw); L2 flushed before every call",
                "steps": r["bwd"]["steps"], "ms": bwd_att_ms + bwd_cmp_ms,
                "attention_backward": {
                    "ms": bwd_att_ms, "tflops": bt, "pct_of_bf16_peak": 100.0 * bt / peak_t,
                    "flops_per_launch": bf, "executed_flops": bx,
                    "executed_tflops": bx / (bwd_att_ms * 1e-3) / 1e12,
                    "roofline": {"bound": "tensor", "achieved": bt, "peak": peak_t, "unit": "TFLOP/s",
                                 "frac": bt / peak_t, "traffic": profile_traffic("backward", wl.name),
                                 "peak_source": f"{peak_src} bf16_tflops (burst)"}},
                "compress_backward": {
                    "ms": bwd_cmp_ms, "gbs": cg, "bytes": cb,
                    "roofline": {"bound": "hbm", "achieved": cg, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": cg / peaks["hbm_gbs"], "traffic": None,
                                 "peak_source": f"{peak_src} hbm_gbs"}},
                "gpu_launches": r["bwd"]["launches"] * r["bwd"]["steps"],
                "cpu_baseline": (backward_cpu_baseline(wl, r["x"], r["bwd"]["gsample"])
                                 if (not args.no_cpu_baseline and world == 1) else None)}
        if r["dec"] is not None:
            dw = r["dec"]["wl"]
            db = decode_bytes(dw)
            dg = db / (dec_ms * 1e-3) / 1e9
            dfl = 2.0 * (dw.d1 + dw.d2) * dw.n1 * dw.n_cmp * dw.batch
            line["paged_decode"] = {
                "what": f"nsa_compress_attention_paged: {dw.batch} sequences x 1 query against {dw.n_cmp} compressed "
                        f"blocks each ({dw.raw_len} raw tokens), N1={dw.n1}, N2={dw.n2}, D={dw.d1}, pages of "
                        f"{dw.page_size} blocks in a permuted pool; L2 flushed before every call",
                "workload": dw.name, "ms": dec_ms, "steps": r["dec"]["steps"],
                "decode_tok_s": world * dw.batch / (dec_ms * 1e-3), "gbs": dg, "bytes": db,
                "tflops": dfl / (dec_ms * 1e-3) / 1e12,
                "roofline": {"bound": "hbm", "achieved": dg, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": dg / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peak_src} hbm_gbs"},
                "gpu_launches": r["dec"]["steps"],
                "cpu_baseline": (decode_cpu_baseline(dw, r["dec"]["x"])
                                 if (not args.no_cpu_baseline and world == 1) else None)}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
