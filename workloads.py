"""Seeded synthetic workloads for the NSA compressed-attention path.

This module only builds inputs: shapes, sequence lengths, random tensors and
hyper-parameters.  It holds none of the method's arithmetic and is shared by
the tests, the benchmark and the smoke check (the oracle and the CUDA path
both consume what it returns).

Recipe (stated once here, repeated in the design notes):
  * q, k, v: ``randn`` in float32 from a ``torch.Generator`` seeded with the
    workload's seed, multiplied by ``std``, then cast to the storage dtype.
    Order of draws: q, k, v, w, then the key-outlier mask when present.
  * w: ``rand * (2 / l)`` (uniform on [0, 2/l)), cast to the storage dtype.
  * key outliers (long-context workload): a Bernoulli(p) mask over
    (token, kv-head) of the raw keys scales those key vectors by ``factor``.
  * cu_sel_kv: prefix sums of ceil(S_b / l') (the number of selection blocks
    of each raw sequence).
  * Short-query workloads keep the last ``q_last`` tokens of each sequence.
  * Backward: the incoming gradient of attention_out is ``randn`` (T1, N1, D2)
    from a generator seeded with seed + 1000, cast to the storage dtype.
The pages name no dataset or benchmark suite; these inputs stand alone.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple           # raw sequence lengths S_b
    n1: int                  # query heads
    n2: int                  # key/value heads
    d1: int                  # query/key head dim
    d2: int                  # value head dim
    l: int                   # compress_block_size
    d: int                   # compress_stride
    lp: int                  # select_block_size
    count: int               # select_block_count
    scale: float
    dtype: str = "bf16"      # "bf16" | "fp16"
    seed: int = 0
    std: float = 1.0
    outlier_p: float = 0.0   # fraction of (token, kv-head) keys scaled by outlier_factor
    outlier_factor: float = 1.0
    q_last: Optional[int] = None  # queries = last q_last tokens of each sequence

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def t2(self) -> int:
        return int(sum(self.seqlens))

    def q_lengths(self) -> List[int]:
        if self.q_last is None:
            return list(self.seqlens)
        return [min(self.q_last, s) for s in self.seqlens]

    def cu_seqlens(self) -> np.ndarray:
        return np.cumsum(np.asarray(self.seqlens, dtype=np.int64)).astype(np.int32)

    def cu_seqlens_q(self) -> np.ndarray:
        return np.cumsum(np.asarray(self.q_lengths(), dtype=np.int64)).astype(np.int32)

    def cu_sel_kv(self) -> np.ndarray:
        nsel = [-(-s // self.lp) for s in self.seqlens]
        return np.cumsum(np.asarray(nsel, dtype=np.int64)).astype(np.int32)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def generate(self, device: str = "cpu"):
        """Return the seeded inputs as a dict of tensors on ``device``.

        Keys: q (T1,N1,D1), k (T2,N2,D1), v (T2,N2,D2), w (l,N2) and the host
        int32 arrays cu_seqlens, cu_seqlens_q, cu_sel_kv.
        """
        g = torch.Generator(device=device)
        g.manual_seed(self.seed)
        dt = self.torch_dtype
        t2 = self.t2
        cu = self.cu_seqlens()
        qlens = self.q_lengths()
        t1_full = t2 if self.q_last is None else None

        def randn(*shape):
            x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
            if self.std != 1.0:
                x.mul_(self.std)
            return x

        if t1_full is not None:
            q = randn(t2, self.n1, self.d1).to(dt)
        else:
            # queries drawn for the whole raw sequence, then the last q_last kept
            qfull = randn(t2, self.n1, self.d1).to(dt)
            parts, start = [], 0
            for s, ql in zip(self.seqlens, qlens):
                parts.append(qfull[start + s - ql:start + s])
                start += s
            q = torch.cat(parts, 0).contiguous()
            del qfull
        kf = randn(t2, self.n2, self.d1)
        v = randn(t2, self.n2, self.d2).to(dt)
        w = (torch.rand(self.l, self.n2, generator=g, device=device,
                        dtype=torch.float32) * (2.0 / self.l)).to(dt)
        if self.outlier_p > 0.0:
            m = torch.rand(t2, self.n2, generator=g, device=device,
                           dtype=torch.float32) < self.outlier_p
            kf = torch.where(m[:, :, None], kf * self.outlier_factor, kf)
        k = kf.to(dt)
        del kf
        return {"q": q, "k": k, "v": v, "w": w, "cu_seqlens": cu,
                "cu_seqlens_q": self.cu_seqlens_q(), "cu_sel_kv": self.cu_sel_kv()}


def grad_output(wl: Workload, device: str = "cpu") -> torch.Tensor:
    """The seeded incoming gradient of attention_out, (T1, N1, D2)."""
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed + 1000)
    t1 = int(sum(wl.q_lengths()))
    return torch.randn(t1, wl.n1, wl.d2, generator=g, device=device, dtype=torch.float32).to(wl.torch_dtype)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One query per sequence against a paged compressed K/V cache."""
    name: str
    batch: int
    raw_len: int            # raw tokens of every sequence
    n1: int
    n2: int
    d1: int
    d2: int
    l: int
    d: int
    lp: int
    count: int
    page_size: int
    scale: float
    dtype: str = "bf16"
    seed: int = 6
    std: float = 0.25       # of the compressed keys and values drawn directly

    @property
    def n_cmp(self) -> int:
        return 0 if self.raw_len < self.l else (self.raw_len - self.l) // self.d + 1

    def generate(self, device: str = "cpu"):
        """q (batch, N1, D1); page pools kcmp / vcmp (pages, page_size, N2, D); a
        block table (batch, pages per sequence) int32 whose pages are a seeded
        permutation of the pool; host prefix sums cu_seqlens_q (1 .. batch),
        cu_cmp_kv and cu_sel_kv.  The compressed cache is drawn directly
        (randn * std): its values play no part in the work done."""
        g = torch.Generator(device=device)
        g.manual_seed(self.seed)
        dt = torch.bfloat16 if self.dtype == "bf16" else torch.float16
        ppseq = -(-self.n_cmp // self.page_size)
        npages = self.batch * ppseq
        q = torch.randn(self.batch, self.n1, self.d1, generator=g, device=device).to(dt)
        kp = (torch.randn(npages, self.page_size, self.n2, self.d1, generator=g, device=device) * self.std).to(dt)
        vp = (torch.randn(npages, self.page_size, self.n2, self.d2, generator=g, device=device) * self.std).to(dt)
        perm = torch.randperm(npages, generator=g, device=device).to(torch.int32)
        table = perm.view(self.batch, ppseq).contiguous()
        b = np.arange(1, self.batch + 1, dtype=np.int64)
        nsel = -(-self.raw_len // self.lp)
        return {"q": q, "kcmp_pages": kp, "vcmp_pages": vp, "block_table": table,
                "cu_seqlens_q": b.astype(np.int32), "cu_cmp_kv": (b * self.n_cmp).astype(np.int32),
                "cu_sel_kv": (b * nsel).astype(np.int32)}


def _varlen_lengths() -> tuple:
    lens = np.random.default_rng(1).integers(2048, 32768, 8, endpoint=True)
    return tuple(int(x) for x in lens)


# The five workloads of the hot-path specification.
TINY = Workload("tiny_s1024_n4_g4_d64", (1024,), 4, 1, 64, 64, 32, 16, 64, 8,
                1.0 / 8.0, "bf16", seed=0)
SINGLE_16K = Workload("single_s16384_n64_n4_d128", (16384,), 64, 4, 128, 128,
                      32, 16, 64, 16, 128 ** -0.5, "bf16", seed=1)
VARLEN_8 = Workload("varlen8_t158963_n32_n2_d192x128_fp16", _varlen_lengths(),
                    32, 2, 192, 128, 64, 32, 64, 16, 192 ** -0.5, "fp16", seed=2)
LONG_128K = Workload("long_s131072_n128_n8_d128", (131072,), 128, 8, 128, 128,
                     64, 32, 128, 32, 128 ** -0.5, "bf16", seed=3, std=0.5,
                     outlier_p=0.02, outlier_factor=4.0)
SHORTQ_4x64K = Workload("compress_t262144_shortq_4x128_n64_n8_d128",
                        (65536,) * 4, 64, 8, 128, 128, 128, 64, 128, 32,
                        128 ** -0.5, "bf16", seed=4, q_last=128)

# A profiling case, not one of the benchmark's configurations: the shape of the
# 16K workload at twice the length (M-tiles visit twice as many KV tiles), with
# a device footprint near 1 GB, small enough for a full ncu capture.
PROFILE_32K = Workload("single_s32768_n64_n4_d128", (32768,), 64, 4, 128, 128,
                       32, 16, 64, 16, 128 ** -0.5, "bf16", seed=5)

# Decode: 64 sequences of 65536 raw tokens (1023 compressed blocks each, the
# short-query workload's block geometry), one query each, 64-block pages.
DECODE_64x64K = DecodeWorkload("decode_b64_s65536_n64_n8_d128_page64", 64, 65536, 64, 8, 128, 128, 128, 64, 128,
                               32, 64, 128 ** -0.5)

WORKLOADS = {w.name: w for w in (TINY, SINGLE_16K, VARLEN_8, LONG_128K, SHORTQ_4x64K, PROFILE_32K)}
BY_INDEX = [TINY, SINGLE_16K, VARLEN_8, LONG_128K, SHORTQ_4x64K]


def sample_rows(cu_seqlens_q: np.ndarray, first: int = 512, last: int = 512,
                every: int = 61) -> np.ndarray:
    """Deterministic query-row sample for workloads too large for the oracle:
    the first and last rows of every sequence plus every ``every``-th row."""
    rows = set()
    prev = 0
    for end in cu_seqlens_q.tolist():
        rows.update(range(prev, min(prev + first, end)))
        rows.update(range(max(prev, end - last), end))
        rows.update(range(prev, end, every))
        prev = end
    return np.asarray(sorted(rows), dtype=np.int64)
