"""fp64 CPU oracle for the NSA compressed-attention path (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never imports it,
and it shares no code with the CUDA path.  The arithmetic lives in
``nsa_oracle.c`` (plain C, fp64, OpenMP over query rows); this module compiles
it with gcc on first use and marshals numpy arrays through ctypes.

Pages followed (cited by title and section):
  * "aclnnNsaCompress" -- Formula section (sliding-window compression).
  * "mindspore.ops.nsa_compress_attention" -- steps 1-7, note list, Returns.
  * "lite_boost.ops.rain_fusion_attention" -- select_idx ordering (ascending,
    then -1 padding).

Parity of the query-offset, top-k candidate, output-order and empty-row
readings is unpinned (no page gives an example for them).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libnsa_oracle.so")
_lib = None
_lock = threading.Lock()

BF16, FP16 = 0, 1

_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile nsa_oracle.c into libnsa_oracle.so next to it (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-std=gnu11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.oracle_round.argtypes = [_f64p, ctypes.c_int64, ctypes.c_int, _f64p]
        lib.oracle_round.restype = None
        lib.oracle_compress_len.argtypes = [_i32p, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, _i32p]
        lib.oracle_compress_len.restype = ctypes.c_int64
        lib.oracle_compress.argtypes = [_f64p, _f64p, ctypes.c_int, ctypes.c_int,
                                        _i32p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, _i32p, _f64p]
        lib.oracle_compress.restype = None
        lib.oracle_importance.argtypes = [_f64p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _f64p]
        lib.oracle_importance.restype = None
        lib.oracle_topk.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _i32p]
        lib.oracle_topk.restype = None
        lib.oracle_compress_attention.argtypes = [
            _f64p, _f64p, _f64p, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _i32p, _i32p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
            _f64p, _f64p, _f64p, _i32p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64]
        lib.oracle_compress_attention.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_select_attention.argtypes = [
            _f64p, _f64p, _f64p, _i32p, ctypes.c_double,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            _i32p, _i32p, ctypes.c_int,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
            _f64p, _f64p]
        lib.oracle_select_attention.restype = ctypes.c_int
        lib.oracle_compress_attention_backward.argtypes = [
            _f64p, _f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _i32p, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_int64, _f64p, _f64p, _f64p]
        lib.oracle_compress_attention_backward.restype = ctypes.c_int
        lib.oracle_compress_backward.argtypes = [
            _f64p, _f64p, _f64p, ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, _f64p, _f64p]
        lib.oracle_compress_backward.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _f64(x) -> np.ndarray:
    """fp64 copy of an array or torch tensor (bf16/fp16 -> fp64 is exact)."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def round_storage(x, dtype: int) -> np.ndarray:
    """Round fp64 values to bfloat16 (dtype 0) or float16 (dtype 1), RNE."""
    xin = _f64(x)
    out = np.empty_like(xin)
    _load().oracle_round(xin.reshape(-1), xin.size, int(dtype), out.reshape(-1))
    return out


def compress_len(cu_seqlens, l: int, d: int) -> np.ndarray:
    """Cumulative compressed lengths (aclnnNsaCompress, Formula section)."""
    cu = _i32(cu_seqlens)
    out = np.empty_like(cu)
    _load().oracle_compress_len(cu, cu.size, int(l), int(d), out)
    return out


def compress(x, w, l: int, d: int, cu_seqlens, dtype: int | None = None):
    """Compress one tensor x (T, N2, D) with weights w (l, N2).

    Returns (out, cu_cmp): out is (Tc, N2, D) fp64, rounded to the storage
    dtype when ``dtype`` is given, else unrounded.
    """
    xf = _f64(x)
    wf = _f64(w)
    cu = _i32(cu_seqlens)
    T, n2, dim = xf.shape
    assert wf.shape == (l, n2)
    cu_cmp = compress_len(cu, l, d)
    tc = int(cu_cmp[-1]) if cu.size else 0
    out = np.zeros((max(tc, 0), n2, dim), dtype=np.float64)
    if tc > 0:
        _load().oracle_compress(xf, wf, int(l), int(d), cu, cu.size, n2, dim,
                                cu_cmp, out)
    if dtype is not None:
        out = round_storage(out, dtype)
    return out, cu_cmp


def importance(P, n_vis: int, a: int, b: int, n_sel: int) -> np.ndarray:
    """Step 4 importance scores of one head row from its probabilities P."""
    pf = _f64(P)
    if pf.size == 0:
        pf = np.zeros(1)
    out = np.empty(max(n_sel, 1), dtype=np.float64)
    _load().oracle_importance(pf, int(n_vis), int(a), int(b), int(n_sel), out)
    return out[:n_sel]


def topk(score, n_cand: int, count: int) -> np.ndarray:
    """Step 7 top-k over candidates 0..n_cand-1 (ascending output, -1 pad)."""
    sf = _f64(score)
    if sf.size == 0:
        sf = np.zeros(1)
    out = np.empty(count, dtype=np.int32)
    _load().oracle_topk(sf, int(n_cand), int(count), out)
    return out


def compress_attention(q, kcmp, vcmp, scale: float, l: int, d: int, lp: int,
                       count: int, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                       rows=None, sel_cap: int | None = None, q_rows_only: bool = False,
                       atten_mask=None, topk_mask=None):
    """Steps 1-7 of mindspore.ops.nsa_compress_attention for query rows.

    q (T1, N1, D1), kcmp (Tc, N2, D1), vcmp (Tc, N2, D2): values of the
    storage-dtype tensors.  ``rows`` selects global query rows (None = all);
    with ``q_rows_only`` q holds just those rows, in the order of ``rows``.
    ``atten_mask`` (S1, S2cmp) and ``topk_mask`` (S1, S2sel), bool, optional:
    one matrix for every sequence and head, indexed by (query index inside the
    sequence, block); True removes the block from the visible set (step 1) or
    from the top-k candidates (step 6).
    Returns a dict with out (R, N1, D2), softmax_max / softmax_sum (R, N1),
    topk (R, N2, count), score (R, N2, sel_cap) and ncand (R, N2).
    """
    qf, kf, vf = _f64(q), _f64(kcmp), _f64(vcmp)
    _, n1, d1 = qf.shape
    tc, n2, d1k = kf.shape
    d2 = vf.shape[2]
    assert d1k == d1 and vf.shape[:2] == (tc, n2)
    cq, cc, cs = _i32(cu_seqlens_q), _i32(cu_cmp_kv), _i32(cu_sel_kv)
    batch = cq.size
    if q_rows_only and rows is None:
        raise ValueError("q_rows_only needs rows")
    if rows is None:
        rows_arr = np.arange(int(cq[-1]) if batch else 0, dtype=np.int64)
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    R = rows_arr.size
    if sel_cap is None:
        nsel = np.diff(np.concatenate([[0], cs])) if batch else np.zeros(1)
        sel_cap = int(max(int(np.max(nsel)) if nsel.size else 1, 1))
    out = np.zeros((R, n1, d2))
    smax = np.zeros((R, n1))
    ssum = np.zeros((R, n1))
    tk = np.zeros((R, n2, count), dtype=np.int32)
    score = np.zeros((R, n2, sel_cap))
    ncand = np.zeros((R, n2), dtype=np.int32)
    if kf.size == 0:
        kf = np.zeros(1)
    if vf.size == 0:
        vf = np.zeros(1)
    def _mask(mk, need_cols, what):
        if mk is None:
            return None, 0
        mk = np.ascontiguousarray(np.asarray(mk).astype(np.uint8))
        seq_q = np.diff(np.concatenate([[0], cq])) if batch else np.zeros(1, np.int64)
        if mk.ndim != 2 or mk.shape[0] < int(np.max(seq_q, initial=0)) or mk.shape[1] < need_cols:
            raise ValueError(f"{what} must be (S1, S2) covering every sequence's queries and blocks")
        return mk, mk.shape[1]
    max_cmp = int(np.max(np.diff(np.concatenate([[0], cc])), initial=0)) if batch else 0
    max_sel = int(np.max(np.diff(np.concatenate([[0], cs])), initial=0)) if batch else 0
    am, am_s2 = _mask(atten_mask, max_cmp, "atten_mask")
    tm, tm_s2 = _mask(topk_mask, max_sel, "topk_mask")
    if R > 0:
        rc = _load().oracle_compress_attention(
            qf, kf, vf, float(scale), n1, n2, d1, d2, int(l), int(d), int(lp),
            int(count), cq, cc, cs, batch,
            rows_arr.ctypes.data_as(ctypes.c_void_p), R, 1 if q_rows_only else 0,
            out, smax, ssum, tk, score.ctypes.data_as(ctypes.c_void_p), sel_cap,
            ncand.ctypes.data_as(ctypes.c_void_p),
            am.ctypes.data_as(ctypes.c_void_p) if am is not None else None, am_s2,
            tm.ctypes.data_as(ctypes.c_void_p) if tm is not None else None, tm_s2)
        if rc != 0:
            raise ValueError("oracle: l % d and l' % d must be 0")
    return {"out": out, "softmax_max": smax, "softmax_sum": ssum, "topk": tk,
            "score": score, "ncand": ncand, "rows": rows_arr}


def select_attention(q, k, v, sel, scale: float, lp: int, count: int, cu_seqlens_q,
                     cu_seqlens_kv, rows=None, q_rows_only: bool = False):
    """Selection attention over the l'-token KV blocks listed per (query row,
    KV group) in ``sel`` ("lite_boost.ops.rain_fusion_attention": index lists,
    causal mask, GQA; fed with the top-k of the compressed branch).

    q (T1, N1, D1), k (T2, N2, D1), v (T2, N2, D2): values of the storage-dtype
    tensors; sel (T1, N2, count) int32 over all query rows.  ``rows`` /
    ``q_rows_only`` as in compress_attention.  Returns a dict with out
    (R, N1, D2) and lse (R, N1).
    """
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    _, n1, d1 = qf.shape
    t2, n2, d1k = kf.shape
    d2 = vf.shape[2]
    assert d1k == d1 and vf.shape[:2] == (t2, n2)
    sl = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    assert sl.shape[1:] == (n2, count)
    cq, ck = _i32(cu_seqlens_q), _i32(cu_seqlens_kv)
    batch = cq.size
    if q_rows_only and rows is None:
        raise ValueError("q_rows_only needs rows")
    if rows is None:
        rows_arr = np.arange(int(cq[-1]) if batch else 0, dtype=np.int64)
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    R = rows_arr.size
    out = np.zeros((R, n1, d2))
    lse = np.zeros((R, n1))
    if kf.size == 0:
        kf = np.zeros(1)
    if vf.size == 0:
        vf = np.zeros(1)
    if sl.size == 0:
        sl = np.zeros(1, dtype=np.int32)
    if R > 0:
        rc = _load().oracle_select_attention(
            qf, kf, vf, sl, float(scale), n1, n2, d1, d2, int(lp), int(count), cq, ck, batch,
            rows_arr.ctypes.data_as(ctypes.c_void_p), R, 1 if q_rows_only else 0, out, lse)
        if rc != 0:
            raise ValueError("oracle: bad selection-attention arguments")
    return {"out": out, "lse": lse, "rows": rows_arr}


def compress_attention_backward(q, kcmp, vcmp, dout, scale: float, l: int, d: int, cu_seqlens_q,
                                cu_cmp_kv, atten_mask=None):
    """Gradient of attention_out (steps 1-3) with respect to q, kcmp and vcmp
    for the incoming dout (T1, N1, D2); the importance scores and the top-k
    carry none.  ``atten_mask`` as in compress_attention.  Returns a dict
    with dq (T1, N1, D1), dkcmp (Tc, N2, D1), dvcmp (Tc, N2, D2), fp64."""
    qf, kf, vf, gf = _f64(q), _f64(kcmp), _f64(vcmp), _f64(dout)
    t1, n1, d1 = qf.shape
    tc, n2, _ = kf.shape
    d2 = vf.shape[2]
    assert gf.shape == (t1, n1, d2)
    cq, cc = _i32(cu_seqlens_q), _i32(cu_cmp_kv)
    am, am_s2 = None, 0
    if atten_mask is not None:
        am = np.ascontiguousarray(np.asarray(atten_mask).astype(np.uint8))
        am_s2 = am.shape[1]
    dq = np.zeros((t1, n1, d1))
    dk = np.zeros((max(tc, 1), n2, d1))
    dv = np.zeros((max(tc, 1), n2, d2))
    rc = _load().oracle_compress_attention_backward(
        qf, kf if kf.size else np.zeros(1), vf if vf.size else np.zeros(1), gf, float(scale), n1, n2, d1, d2,
        int(l), int(d), cq, cc, cq.size, am.ctypes.data_as(ctypes.c_void_p) if am is not None else None,
        am_s2, dq, dk, dv)
    if rc != 0:
        raise ValueError("oracle: N1 must be a multiple of N2")
    return {"dq": dq, "dkcmp": dk[:tc], "dvcmp": dv[:tc]}


def compress_backward(x, w, dcmp, l: int, d: int, cu_seqlens):
    """Gradient of the compression of x (T, N2, D) with weights w (l, N2) for
    the incoming dcmp (Tc, N2, D).  Returns (dx (T, N2, D), dw (l, N2)), fp64."""
    xf, wf, gf = _f64(x), _f64(w), _f64(dcmp)
    T, n2, dim = xf.shape
    cu = _i32(cu_seqlens)
    dx = np.zeros((T, n2, dim))
    dw = np.zeros((l, n2))
    _load().oracle_compress_backward(xf, wf, gf if gf.size else np.zeros(1), int(l), int(d), cu, cu.size, n2,
                                     dim, dx, dw)
    return dx, dw
