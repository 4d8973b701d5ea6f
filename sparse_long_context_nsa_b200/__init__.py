"""B200-native NSA compressed-attention path: Python binding of libnsa_b200.so.

This module only marshals arguments: every step of the computation runs in
the CUDA kernels of the C-ABI library (``include/nsa.h``).  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: importing
works without a GPU (for the host-only entry points), and every device entry
point raises when the library or a CUDA device is missing.

Entry points (same names as the C ABI):
  nsa_compress_out_len, nsa_compress, nsa_compress_attention_workspace_size,
  nsa_compress_attention, nsa_compress_attention_noalloc, nsa_select_attention,
  nsa_workspace_status, nsa_compress_status, nsa_noalloc_status,
  nsa_status_string.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnsa_b200.so")
# NSA_DEBUG=1: load the debug build (device bounds checks) and put a guard band
# with a canary pattern after every output and workspace this binding allocates,
# checked after every call.
LIB_DEBUG_PATH = os.path.join(_PKG, "libnsa_b200_debug.so")
DEBUG = os.environ.get("NSA_DEBUG") == "1"
_GUARD_BYTES = 4096
_CANARY = 0xA5
_guards = []   # (name, guard bytes) of the allocations made for the current call

NSA_OK, NSA_ERR_INVALID_ARG, NSA_ERR_UNSUPPORTED = 0, 1, 2
NSA_ERR_WORKSPACE, NSA_ERR_CUDA, NSA_ERR_TIMEOUT = 3, 4, 5
NSA_BF16, NSA_FP16 = 0, 1

EXPORTED = (
    "nsa_status_string",
    "nsa_compress_out_len",
    "nsa_compress",
    "nsa_compress_attention_workspace_size",
    "nsa_compress_attention",
    "nsa_compress_attention_masked",
    "nsa_compress_attention_masked_workspace_size",
    "nsa_compress_attention_paged",
    "nsa_compress_paged",
    "nsa_workspace_status",
    "nsa_compress_status",
    "nsa_compress_attention_noalloc",
    "nsa_noalloc_status",
    "nsa_select_attention_workspace_size",
    "nsa_select_attention",
    "nsa_shard_groups",
    "nsa_compress_attention_shard_workspace_size",
    "nsa_compress_attention_shard",
    "nsa_compress_attention_shard_plan",
    "nsa_compress_attention_backward_workspace_size",
    "nsa_compress_attention_backward",
    "nsa_compress_backward_workspace_size",
    "nsa_compress_backward",
)

_lib = None


class NsaError(RuntimeError):
    """A CUDA failure, a device-side timeout or a workspace problem."""

    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_status_name(status)}")
        self.status = status


def _status_name(status: int) -> str:
    try:
        return load().nsa_status_string(status).decode()
    except Exception:  # library missing: still report the number
        return f"status {status}"


def load(path: Optional[str] = None):
    """Load the C-ABI library (built in-tree); raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or (LIB_DEBUG_PATH if DEBUG else LIB_PATH)
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with sparse_long_context_nsa_b200._build.build()")
    lib = ctypes.CDLL(p)
    i32p = ctypes.POINTER(ctypes.c_int32)
    vp, ci, cs = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.nsa_status_string.argtypes = [ci]
    lib.nsa_status_string.restype = ctypes.c_char_p
    lib.nsa_compress_out_len.argtypes = [i32p, ci, ci, ci, i32p, ctypes.POINTER(ctypes.c_int64)]
    lib.nsa_compress_out_len.restype = ci
    lib.nsa_compress.argtypes = [vp, vp, vp, ci, ci, i32p, ci, ci, ci, ci, ci, vp, vp, vp]
    lib.nsa_compress.restype = ci
    lib.nsa_compress_attention_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, i32p, i32p,
                                                          i32p, ci, ctypes.POINTER(cs)]
    lib.nsa_compress_attention_workspace_size.restype = ci
    lib.nsa_compress_attention.argtypes = [vp, vp, vp, ctypes.c_float, ci, ci, ci, ci, ci, i32p, i32p,
                                           i32p, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, cs, vp]
    lib.nsa_compress_attention.restype = ci
    lib.nsa_compress_attention_masked.argtypes = [vp, vp, vp, ctypes.c_float, ci, ci, ci, ci, ci, i32p, i32p,
                                                  i32p, ci, ci, ci, ci, ci, vp, ci, ci, vp, ci, ci, vp, vp, vp,
                                                  vp, vp, cs, vp]
    lib.nsa_compress_attention_masked.restype = ci
    lib.nsa_compress_attention_masked_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, i32p, i32p, i32p,
                                                                 ci, ci, ci, ctypes.POINTER(ctypes.c_size_t)]
    lib.nsa_compress_attention_masked_workspace_size.restype = ci
    lib.nsa_compress_attention_paged.argtypes = [vp, vp, vp, ctypes.c_int64, ci, vp, ci, ctypes.c_float, ci, ci, ci,
                                                 ci, ci, i32p, i32p, i32p, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp,
                                                 ctypes.c_size_t, vp]
    lib.nsa_compress_attention_paged.restype = ci
    lib.nsa_compress_paged.argtypes = [vp, vp, vp, ci, ci, i32p, ci, ci, ci, ci, ci, vp, vp, ctypes.c_int64, ci, vp,
                                       ci, i32p, vp]
    lib.nsa_compress_paged.restype = ci
    lib.nsa_workspace_status.argtypes = [vp, vp]
    lib.nsa_workspace_status.restype = ci
    lib.nsa_compress_status.argtypes = [vp]
    lib.nsa_compress_status.restype = ci
    lib.nsa_compress_attention_noalloc.argtypes = [vp, vp, vp, ctypes.c_float, ci, ci, ci, ci, ci, i32p,
                                                   i32p, i32p, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp]
    lib.nsa_compress_attention_noalloc.restype = ci
    lib.nsa_noalloc_status.argtypes = [vp]
    lib.nsa_noalloc_status.restype = ci
    lib.nsa_select_attention_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, i32p, i32p, ci,
                                                        ctypes.POINTER(cs)]
    lib.nsa_select_attention_workspace_size.restype = ci
    lib.nsa_select_attention.argtypes = [vp, vp, vp, vp, ctypes.c_float, ci, ci, ci, i32p, i32p, ci, ci, ci,
                                         ci, ci, vp, vp, vp, cs, vp]
    lib.nsa_select_attention.restype = ci
    lib.nsa_shard_groups.argtypes = [ci, ci, ci, ctypes.POINTER(ci), ctypes.POINTER(ci)]
    lib.nsa_shard_groups.restype = ci
    lib.nsa_compress_attention_shard_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, i32p, i32p, i32p,
                                                                ci, ci, ci, ctypes.POINTER(cs)]
    lib.nsa_compress_attention_shard_workspace_size.restype = ci
    lib.nsa_compress_attention_shard.argtypes = [vp, vp, vp, ctypes.c_float, ci, ci, ci, ci, ci, i32p, i32p, i32p,
                                                 ci, ci, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, cs, vp]
    lib.nsa_compress_attention_shard.restype = ci
    lib.nsa_compress_attention_shard_plan.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, i32p, i32p, i32p, ci, ci, ci,
                                                      vp, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
    lib.nsa_compress_attention_shard_plan.restype = ci
    lib.nsa_compress_attention_backward_workspace_size.argtypes = [ci, ci, ci, ci, ci, ci, i32p, i32p, ci,
                                                                   ctypes.POINTER(ctypes.c_size_t)]
    lib.nsa_compress_attention_backward_workspace_size.restype = ci
    lib.nsa_compress_attention_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, ci, ci, ci, i32p,
                                                    i32p, ci, ci, ci, ci, ci, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.nsa_compress_attention_backward.restype = ci
    lib.nsa_compress_backward_workspace_size.argtypes = [i32p, ci, ci, ci, ctypes.POINTER(ctypes.c_size_t)]
    lib.nsa_compress_backward_workspace_size.restype = ci
    lib.nsa_compress_backward.argtypes = [vp, vp, vp, vp, vp, ci, ci, i32p, ci, ci, ci, ci, ci, vp, vp, vp, vp,
                                          ctypes.c_size_t, vp]
    lib.nsa_compress_backward.restype = ci
    if path is None:
        _lib = lib
    return lib


def _alloc(fill, *shape, dtype, device) -> torch.Tensor:
    """An output or workspace tensor; in debug mode followed by a guard band of
    canary bytes that _raise checks once the call has run."""
    if not DEBUG:
        return (torch.zeros if fill else torch.empty)(*shape, dtype=dtype, device=device)
    n = 1
    for x in shape:
        n *= int(x)
    esize = torch.empty((), dtype=dtype).element_size()
    flat = torch.empty(n * esize + _GUARD_BYTES, dtype=torch.uint8, device=device)
    if fill:
        flat[:n * esize].zero_()
    flat[n * esize:].fill_(_CANARY)
    _guards.append((f"{tuple(shape)} {dtype}", flat[n * esize:]))
    return flat[:n * esize].view(dtype).view(*shape)


def _empty(*shape, dtype, device) -> torch.Tensor:
    return _alloc(False, *shape, dtype=dtype, device=device)


def _zeros(*shape, dtype, device) -> torch.Tensor:
    return _alloc(True, *shape, dtype=dtype, device=device)


def _check_guards(what: str):
    """Debug mode: every guard band allocated for this call still holds its
    canary pattern (a write past the end of an output would have changed it)."""
    if not _guards:
        return
    torch.cuda.synchronize()
    bad = [name for name, g in _guards if not bool((g == _CANARY).all())]
    _guards.clear()
    if bad:
        raise NsaError(NSA_ERR_INVALID_ARG, f"{what}: guard band overwritten after {', '.join(bad)}")


def _raise(status: int, what: str, guards: bool = False):
    """Maps a status to an exception; after a compute call (guards=True) also
    checks the debug guard bands of the call's allocations."""
    if guards:
        if status == NSA_OK:
            _check_guards(what)
        _guards.clear()
    if status == NSA_OK:
        return
    if status in (NSA_ERR_INVALID_ARG, NSA_ERR_UNSUPPORTED):
        raise ValueError(f"{what}: {_status_name(status)}")
    raise NsaError(status, what)


def _cu(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x.cpu() if hasattr(x, "cpu") else x, dtype=np.int32))
    if a.ndim != 1 or a.size < 1:
        raise ValueError("sequence lengths must be a non-empty 1-D list of prefix sums")
    return a


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return NSA_BF16
    if t.dtype == torch.float16:
        return NSA_FP16
    raise TypeError(f"dtype must be bfloat16 or float16, got {t.dtype}")


def _same_device(ref: torch.Tensor, *named) -> None:
    for t, name in named:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} must be on {ref.device}")


def _out(t: torch.Tensor, shape, dtype, device, name: str) -> torch.Tensor:
    """A caller-provided output: the kernels write exactly this shape, so
    anything else is refused before the launch."""
    _dev(t, name)
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {tuple(shape)} {dtype}, got {tuple(t.shape)} {t.dtype}")
    return t


def _workspace(ws: torch.Tensor, nbytes: int, device) -> torch.Tensor:
    """The caller's workspace, checked; a fresh one only when none is given.

    A caller-provided workspace that is too small is refused rather than
    replaced: the kernel writes its error word into the workspace it runs
    on, and the caller reads that word back from its own tensor."""
    if ws is None:
        return _empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    _dev(ws, "workspace")
    if ws.device != device or ws.dtype != torch.uint8:
        raise ValueError(f"workspace must be a uint8 tensor on {device}")
    if ws.numel() < nbytes:
        raise ValueError(f"workspace holds {ws.numel()} bytes; this call needs {nbytes}")
    return ws


def _dev(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library computes on the GPU only)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (TND layout)")
    return t


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def nsa_status_string(status: int) -> str:
    return load().nsa_status_string(int(status)).decode()


def nsa_compress_out_len(cu_seqlens: Sequence[int], l: int, d: int) -> np.ndarray:
    """Cumulative compressed lengths of the sequences (host)."""
    cu = _cu(cu_seqlens)
    out = np.empty_like(cu)
    tot = ctypes.c_int64(0)
    _raise(load().nsa_compress_out_len(_ip(cu), cu.size, int(l), int(d), _ip(out), ctypes.byref(tot)),
           "nsa_compress_out_len")
    return out


def nsa_compress(k: torch.Tensor, v: Optional[torch.Tensor], w: torch.Tensor, l: int, d: int,
                 cu_seqlens: Sequence[int], kcmp: Optional[torch.Tensor] = None,
                 vcmp: Optional[torch.Tensor] = None, stream=None):
    """Compress raw K (and V) of shape (T2, N2, D) with weights w (l, N2).

    Returns (kcmp, vcmp) of shape (Tc, N2, D); vcmp is None when v is None.
    """
    _dev(k, "k")
    _dev(w, "w")
    dt = _dtype_code(k)
    if w.dtype != k.dtype or (v is not None and v.dtype != k.dtype):
        raise TypeError("k, v and w must share one dtype")
    if k.dim() != 3 or w.dim() != 2:
        raise ValueError("k must be (T2, N2, D1) and w (l, N2)")
    t2, n2, d1 = k.shape
    d2 = d1
    _same_device(k, (w, "w"), (v, "v"))
    if v is not None:
        _dev(v, "v")
        if v.dim() != 3 or v.shape[:2] != k.shape[:2]:
            raise ValueError("v must be (T2, N2, D2) with the T2, N2 of k")
        d2 = v.shape[2]
    if tuple(w.shape) != (l, n2):
        raise ValueError("w must have shape (l, N2)")
    cu = _cu(cu_seqlens)
    if int(cu[-1]) > t2:
        raise ValueError("cu_seqlens runs past the rows of k")
    cuc = nsa_compress_out_len(cu, l, d)
    tc = int(cuc[-1])
    if kcmp is None:
        kcmp = _empty(tc, n2, d1, dtype=k.dtype, device=k.device)
    else:
        _out(kcmp, (tc, n2, d1), k.dtype, k.device, "kcmp")
    if v is not None and vcmp is None:
        vcmp = _empty(tc, n2, d2, dtype=k.dtype, device=k.device)
    elif v is not None:
        _out(vcmp, (tc, n2, d2), k.dtype, k.device, "vcmp")
    st = load().nsa_compress(k.data_ptr(), v.data_ptr() if v is not None else None, w.data_ptr(),
                             int(l), int(d), _ip(cu), cu.size, n2, d1, d2, dt, kcmp.data_ptr(),
                             vcmp.data_ptr() if v is not None else None, _stream(stream))
    _raise(st, "nsa_compress", guards=True)
    return kcmp, vcmp


def nsa_compress_attention_workspace_size(head_num: int, n2: int, d1: int, d2: int, l: int, d: int,
                                          lp: int, count: int, cu_seqlens_q, cu_cmp_kv,
                                          cu_sel_kv) -> int:
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    out = ctypes.c_size_t(0)
    _raise(load().nsa_compress_attention_workspace_size(
        int(head_num), int(n2), int(d1), int(d2), int(l), int(d), int(lp), int(count), _ip(cq), _ip(cc),
        _ip(cs), cq.size, ctypes.byref(out)), "nsa_compress_attention_workspace_size")
    return int(out.value)


def nsa_compress_attention_masked_workspace_size(head_num: int, n2: int, d1: int, d2: int, l: int, d: int,
                                                 lp: int, count: int, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                                 atten_mask: bool = True, topk_mask: bool = True) -> int:
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    out = ctypes.c_size_t(0)
    _raise(load().nsa_compress_attention_masked_workspace_size(
        int(head_num), int(n2), int(d1), int(d2), int(l), int(d), int(lp), int(count), _ip(cq), _ip(cc),
        _ip(cs), cq.size, int(bool(atten_mask)), int(bool(topk_mask)), ctypes.byref(out)),
        "nsa_compress_attention_masked_workspace_size")
    return int(out.value)


def nsa_compress_attention(q: torch.Tensor, kcmp: torch.Tensor, vcmp: torch.Tensor, scale: float,
                           head_num: int, l: int, d: int, lp: int, count: int, cu_seqlens_q,
                           cu_cmp_kv, cu_sel_kv, out=None, workspace: Optional[torch.Tensor] = None,
                           stream=None, atten_mask: Optional[torch.Tensor] = None,
                           topk_mask: Optional[torch.Tensor] = None):
    """Compressed attention + importance scores + top-k.

    Returns (attention_out (T1,N1,D2), topk_indices (T1,N2,count) int32,
    softmax_max (T1,N1,8) fp32, softmax_sum (T1,N1,8) fp32).
    ``out`` may pass these four tensors preallocated.  ``atten_mask``
    (S1, S2cmp) and ``topk_mask`` (S1, S2sel), bool or uint8 device tensors,
    are the page's optional masks: True removes the (query, block) pair, one
    matrix for every sequence and head, row = query index inside the sequence.
    """
    for t, nm in ((q, "q"), (kcmp, "kcmp"), (vcmp, "vcmp")):
        _dev(t, nm)
        if t.dim() != 3:
            raise ValueError(f"{nm} must be 3-D (TND)")
    dt = _dtype_code(q)
    if kcmp.dtype != q.dtype or vcmp.dtype != q.dtype:
        raise TypeError("q, kcmp and vcmp must share one dtype")
    t1, n1, d1 = q.shape
    tc, n2, d1k = kcmp.shape
    d2 = vcmp.shape[2]
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    if d1k != d1 or tuple(vcmp.shape[:2]) != (tc, n2):
        raise ValueError("kcmp must be (Tc, N2, D1) and vcmp (Tc, N2, D2)")
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    if int(cq[-1]) > t1 or int(cc[-1]) > tc:
        raise ValueError("prefix sums run past the rows of q / kcmp")
    dev = q.device
    _same_device(q, (kcmp, "kcmp"), (vcmp, "vcmp"))
    if out is None:
        att = _empty(t1, n1, d2, dtype=q.dtype, device=dev)
        tk = _empty(t1, n2, count, dtype=torch.int32, device=dev)
        smax = _empty(t1, n1, 8, dtype=torch.float32, device=dev)
        ssum = _empty(t1, n1, 8, dtype=torch.float32, device=dev)
    else:
        att, tk, smax, ssum = out
        _out(att, (t1, n1, d2), q.dtype, dev, "attention_out")
        _out(tk, (t1, n2, count), torch.int32, dev, "topk_indices")
        _out(smax, (t1, n1, 8), torch.float32, dev, "softmax_max")
        _out(ssum, (t1, n1, 8), torch.float32, dev, "softmax_sum")
    if atten_mask is None and topk_mask is None:
        ws_bytes = nsa_compress_attention_workspace_size(n1, n2, d1, d2, l, d, lp, count, cq, cc, cs)
    else:
        ws_bytes = nsa_compress_attention_masked_workspace_size(n1, n2, d1, d2, l, d, lp, count, cq, cc, cs,
                                                                atten_mask is not None, topk_mask is not None)
    workspace = _workspace(workspace, ws_bytes, dev)
    if atten_mask is None and topk_mask is None:
        st = load().nsa_compress_attention(
            q.data_ptr(), kcmp.data_ptr(), vcmp.data_ptr(), float(scale), int(head_num), int(l), int(d),
            int(lp), int(count), _ip(cq), _ip(cc), _ip(cs), cq.size, n2, d1, d2, dt, att.data_ptr(),
            tk.data_ptr(), smax.data_ptr(), ssum.data_ptr(), workspace.data_ptr(), workspace.numel(),
            _stream(stream))
        _raise(st, "nsa_compress_attention", guards=True)
        return att, tk, smax, ssum
    masks = []
    for mk, nm in ((atten_mask, "atten_mask"), (topk_mask, "topk_mask")):
        if mk is None:
            masks.append((None, 0, 0))
            continue
        _dev(mk, nm)
        if mk.device != q.device:
            raise ValueError(f"{nm} must be on the device of q")
        if mk.dim() != 2 or mk.dtype not in (torch.bool, torch.uint8) or not mk.is_contiguous():
            raise TypeError(f"{nm} must be a contiguous 2-D bool or uint8 tensor (S1, S2)")
        masks.append((mk, int(mk.shape[0]), int(mk.shape[1])))
    (am, ar, ac), (tm, tr, tc_) = masks
    st = load().nsa_compress_attention_masked(
        q.data_ptr(), kcmp.data_ptr(), vcmp.data_ptr(), float(scale), int(head_num), int(l), int(d),
        int(lp), int(count), _ip(cq), _ip(cc), _ip(cs), cq.size, n2, d1, d2, dt,
        am.data_ptr() if am is not None else None, ar, ac, tm.data_ptr() if tm is not None else None, tr, tc_,
        att.data_ptr(), tk.data_ptr(), smax.data_ptr(), ssum.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream(stream))
    _raise(st, "nsa_compress_attention_masked", guards=True)
    return att, tk, smax, ssum


def nsa_compress_attention_noalloc(q: torch.Tensor, kcmp: torch.Tensor, vcmp: torch.Tensor, scale: float,
                                   head_num: int, l: int, d: int, lp: int, count: int, cu_seqlens_q,
                                   cu_cmp_kv, cu_sel_kv, out, stream=None):
    """nsa_compress_attention for callers that cannot allocate device memory.

    The caller passes the four output tensors in ``out`` (attention_out,
    topk_indices, softmax_max, softmax_sum); the library's own fixed 16 MiB
    scratch array replaces the workspace.  Nothing is allocated here.
    """
    for t, nm in ((q, "q"), (kcmp, "kcmp"), (vcmp, "vcmp")):
        _dev(t, nm)
        if t.dim() != 3:
            raise ValueError(f"{nm} must be 3-D (TND)")
    _same_device(q, (kcmp, "kcmp"), (vcmp, "vcmp"))
    dt = _dtype_code(q)
    if kcmp.dtype != q.dtype or vcmp.dtype != q.dtype:
        raise TypeError("q, kcmp and vcmp must share one dtype")
    t1, n1, d1 = q.shape
    tc, n2, d1k = kcmp.shape
    d2 = vcmp.shape[2]
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    if d1k != d1 or tuple(vcmp.shape[:2]) != (tc, n2):
        raise ValueError("kcmp must be (Tc, N2, D1) and vcmp (Tc, N2, D2)")
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    if int(cq[-1]) > t1 or int(cc[-1]) > tc:
        raise ValueError("prefix sums run past the rows of q / kcmp")
    att, tk, smax, ssum = out
    _out(att, (t1, n1, d2), q.dtype, q.device, "attention_out")
    _out(tk, (t1, n2, count), torch.int32, q.device, "topk_indices")
    _out(smax, (t1, n1, 8), torch.float32, q.device, "softmax_max")
    _out(ssum, (t1, n1, 8), torch.float32, q.device, "softmax_sum")
    st = load().nsa_compress_attention_noalloc(
        q.data_ptr(), kcmp.data_ptr(), vcmp.data_ptr(), float(scale), int(head_num), int(l), int(d),
        int(lp), int(count), _ip(cq), _ip(cc), _ip(cs), cq.size, n2, d1, d2, dt, att.data_ptr(),
        tk.data_ptr(), smax.data_ptr(), ssum.data_ptr(), _stream(stream))
    _raise(st, "nsa_compress_attention_noalloc", guards=True)
    return att, tk, smax, ssum


def nsa_workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and read the device error word of an attention workspace."""
    return int(load().nsa_workspace_status(workspace.data_ptr(), _stream(stream)))


def nsa_compress_status(stream=None) -> int:
    return int(load().nsa_compress_status(_stream(stream)))


def nsa_noalloc_status(stream=None) -> int:
    """Synchronise and read the device error word of the last
    nsa_compress_attention_noalloc on the current device."""
    return int(load().nsa_noalloc_status(_stream(stream)))


def nsa_select_attention_workspace_size(head_num: int, n2: int, d1: int, d2: int, lp: int, count: int,
                                        cu_seqlens_q, cu_seqlens_kv) -> int:
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_kv)
    if cq.size != ck.size:
        raise ValueError("the two prefix-sum lists need one entry per sequence")
    out = ctypes.c_size_t(0)
    _raise(load().nsa_select_attention_workspace_size(
        int(head_num), int(n2), int(d1), int(d2), int(lp), int(count), _ip(cq), _ip(ck), cq.size,
        ctypes.byref(out)), "nsa_select_attention_workspace_size")
    return int(out.value)


def nsa_select_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, topk_indices: torch.Tensor,
                         scale: float, head_num: int, lp: int, cu_seqlens_q, cu_seqlens_kv, out=None,
                         workspace: Optional[torch.Tensor] = None, stream=None):
    """Attention over the l'-token K/V blocks listed in ``topk_indices``
    (T1, N2, count) int32, as written by nsa_compress_attention.

    Returns (attention_out (T1,N1,D2), softmax_lse (T1,N1) fp32); ``out`` may
    pass both preallocated.
    """
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (topk_indices, "topk_indices")):
        _dev(t, nm)
        if t.dim() != 3:
            raise ValueError(f"{nm} must be 3-D")
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share one dtype")
    if topk_indices.dtype != torch.int32 or not topk_indices.is_contiguous():
        raise TypeError("topk_indices must be a contiguous int32 tensor")
    t1, n1, d1 = q.shape
    t2, n2, d1k = k.shape
    d2 = v.shape[2]
    count = topk_indices.shape[2]
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    if d1k != d1 or tuple(v.shape[:2]) != (t2, n2):
        raise ValueError("k must be (T2, N2, D1) and v (T2, N2, D2)")
    if tuple(topk_indices.shape[:2]) != (t1, n2):
        raise ValueError("topk_indices must be (T1, N2, count)")
    cq, ck = _cu(cu_seqlens_q), _cu(cu_seqlens_kv)
    if cq.size != ck.size:
        raise ValueError("the two prefix-sum lists need one entry per sequence")
    if int(cq[-1]) > t1 or int(ck[-1]) > t2:
        raise ValueError("prefix sums run past the rows of q / k")
    dev = q.device
    _same_device(q, (k, "k"), (v, "v"), (topk_indices, "topk_indices"))
    if out is None:
        att = _empty(t1, n1, d2, dtype=q.dtype, device=dev)
        lse = _empty(t1, n1, dtype=torch.float32, device=dev)
    else:
        att, lse = out
        _out(att, (t1, n1, d2), q.dtype, dev, "attention_out")
        _out(lse, (t1, n1), torch.float32, dev, "softmax_lse")
    ws_bytes = nsa_select_attention_workspace_size(n1, n2, d1, d2, lp, count, cq, ck)
    workspace = _workspace(workspace, ws_bytes, dev)
    st = load().nsa_select_attention(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), topk_indices.data_ptr(), float(scale), int(head_num),
        int(lp), int(count), _ip(cq), _ip(ck), cq.size, n2, d1, d2, dt, att.data_ptr(), lse.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream))
    _raise(st, "nsa_select_attention", guards=True)
    return att, lse


# ------------------------------------------------------------ head-group shards
def nsa_shard_groups(n2: int, world: int, rank: int):
    """(group_begin, group_count) of `rank` in the balanced contiguous split of
    n2 KV groups over `world` ranks."""
    b, c = ctypes.c_int(0), ctypes.c_int(0)
    _raise(load().nsa_shard_groups(int(n2), int(world), int(rank), ctypes.byref(b), ctypes.byref(c)),
           "nsa_shard_groups")
    return int(b.value), int(c.value)


def nsa_compress_attention_shard_workspace_size(head_num: int, n2: int, d1: int, d2: int, l: int, d: int, lp: int,
                                                count: int, cu_seqlens_q, cu_cmp_kv, cu_sel_kv,
                                                group_begin: int, group_count: int) -> int:
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    out = ctypes.c_size_t(0)
    _raise(load().nsa_compress_attention_shard_workspace_size(
        int(head_num), int(n2), int(d1), int(d2), int(l), int(d), int(lp), int(count), _ip(cq), _ip(cc), _ip(cs),
        cq.size, int(group_begin), int(group_count), ctypes.byref(out)),
        "nsa_compress_attention_shard_workspace_size")
    return int(out.value)


def nsa_compress_attention_shard_plan(head_num: int, n2: int, d1: int, d2: int, l: int, d: int, lp: int,
                                      count: int, cu_seqlens_q, cu_cmp_kv, cu_sel_kv, group_begin: int,
                                      group_count: int) -> np.ndarray:
    """Work items of a shard's launch, (n_items, 3) int32: first query row,
    tokens, KV group.  Host only."""
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    args = (int(head_num), int(n2), int(d1), int(d2), int(l), int(d), int(lp), int(count), _ip(cq), _ip(cc),
            _ip(cs), cq.size, int(group_begin), int(group_count))
    n = ctypes.c_int64(0)
    _raise(load().nsa_compress_attention_shard_plan(*args, None, 0, ctypes.byref(n)),
           "nsa_compress_attention_shard_plan")
    items = np.zeros((max(int(n.value), 1), 3), dtype=np.int32)
    _raise(load().nsa_compress_attention_shard_plan(*args, items.ctypes.data_as(ctypes.c_void_p), int(n.value),
                                                    ctypes.byref(n)), "nsa_compress_attention_shard_plan")
    return items[:int(n.value)]


def nsa_compress_attention_shard(q: torch.Tensor, kcmp: torch.Tensor, vcmp: torch.Tensor, scale: float,
                                 head_num: int, l: int, d: int, lp: int, count: int, cu_seqlens_q, cu_cmp_kv,
                                 cu_sel_kv, group_begin: int, group_count: int, out=None,
                                 workspace: Optional[torch.Tensor] = None, stream=None):
    """nsa_compress_attention for the KV groups [group_begin, group_begin +
    group_count) only.  Tensors are the whole problem's; the shard's heads are
    read and the shard's outputs written (``out`` may pass the four output
    tensors; rows of other groups are left as they are)."""
    for t, nm in ((q, "q"), (kcmp, "kcmp"), (vcmp, "vcmp")):
        _dev(t, nm)
        if t.dim() != 3:
            raise ValueError(f"{nm} must be 3-D (TND)")
    dt = _dtype_code(q)
    if kcmp.dtype != q.dtype or vcmp.dtype != q.dtype:
        raise TypeError("q, kcmp and vcmp must share one dtype")
    t1, n1, d1 = q.shape
    tc, n2, d1k = kcmp.shape
    d2 = vcmp.shape[2]
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    if d1k != d1 or tuple(vcmp.shape[:2]) != (tc, n2):
        raise ValueError("kcmp must be (Tc, N2, D1) and vcmp (Tc, N2, D2)")
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size):
        raise ValueError("the three prefix-sum lists need one entry per sequence")
    if int(cq[-1]) > t1 or int(cc[-1]) > tc:
        raise ValueError("prefix sums run past the rows of q / kcmp")
    dev = q.device
    _same_device(q, (kcmp, "kcmp"), (vcmp, "vcmp"))
    if out is None:
        att = _zeros(t1, n1, d2, dtype=q.dtype, device=dev)
        tk = torch.full((t1, n2, count), -1, dtype=torch.int32, device=dev)
        smax = _zeros(t1, n1, 8, dtype=torch.float32, device=dev)
        ssum = _zeros(t1, n1, 8, dtype=torch.float32, device=dev)
    else:
        att, tk, smax, ssum = out
        _out(att, (t1, n1, d2), q.dtype, dev, "attention_out")
        _out(tk, (t1, n2, count), torch.int32, dev, "topk_indices")
        _out(smax, (t1, n1, 8), torch.float32, dev, "softmax_max")
        _out(ssum, (t1, n1, 8), torch.float32, dev, "softmax_sum")
    ws_bytes = nsa_compress_attention_shard_workspace_size(n1, n2, d1, d2, l, d, lp, count, cq, cc, cs,
                                                           group_begin, group_count)
    workspace = _workspace(workspace, ws_bytes, dev)
    st = load().nsa_compress_attention_shard(
        q.data_ptr(), kcmp.data_ptr(), vcmp.data_ptr(), float(scale), int(head_num), int(l), int(d), int(lp),
        int(count), _ip(cq), _ip(cc), _ip(cs), cq.size, n2, d1, d2, dt, int(group_begin), int(group_count),
        att.data_ptr(), tk.data_ptr(), smax.data_ptr(), ssum.data_ptr(), workspace.data_ptr(), workspace.numel(),
        _stream(stream))
    _raise(st, "nsa_compress_attention_shard", guards=True)
    return att, tk, smax, ssum


def nsa_compress_attention_backward_workspace_size(head_num: int, n2: int, d1: int, d2: int, l: int, d: int,
                                                   cu_seqlens_q, cu_cmp_kv) -> int:
    cq, cc = _cu(cu_seqlens_q), _cu(cu_cmp_kv)
    if cq.size != cc.size:
        raise ValueError("the prefix-sum lists need one entry per sequence")
    out = ctypes.c_size_t(0)
    _raise(load().nsa_compress_attention_backward_workspace_size(
        int(head_num), int(n2), int(d1), int(d2), int(l), int(d), _ip(cq), _ip(cc), cq.size, ctypes.byref(out)),
        "nsa_compress_attention_backward_workspace_size")
    return int(out.value)


def nsa_compress_attention_backward(q: torch.Tensor, kcmp: torch.Tensor, vcmp: torch.Tensor,
                                    attention_out: torch.Tensor, dout: torch.Tensor, softmax_max: torch.Tensor,
                                    softmax_sum: torch.Tensor, scale: float, head_num: int, l: int, d: int,
                                    cu_seqlens_q, cu_cmp_kv, grads=None, workspace: Optional[torch.Tensor] = None,
                                    stream=None):
    """Gradient of attention_out of nsa_compress_attention with respect to q,
    kcmp and vcmp for the incoming ``dout``, from the forward's inputs, output
    and statistics.  Returns (dq (T1,N1,D1), dkcmp (Tc,N2,D1), dvcmp
    (Tc,N2,D2)), fp32; ``grads`` may pass the three tensors preallocated."""
    for t, nm in ((q, "q"), (kcmp, "kcmp"), (vcmp, "vcmp"), (attention_out, "attention_out"), (dout, "dout")):
        _dev(t, nm)
        if t.dim() != 3:
            raise ValueError(f"{nm} must be 3-D (TND)")
    dt = _dtype_code(q)
    for t, nm in ((kcmp, "kcmp"), (vcmp, "vcmp"), (attention_out, "attention_out"), (dout, "dout")):
        if t.dtype != q.dtype:
            raise TypeError(f"{nm} must have the dtype of q")
    t1, n1, d1 = q.shape
    tc, n2, _ = kcmp.shape
    d2 = vcmp.shape[2]
    dev = q.device
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    if kcmp.shape[2] != d1 or tuple(vcmp.shape[:2]) != (tc, n2):
        raise ValueError("kcmp must be (Tc, N2, D1) and vcmp (Tc, N2, D2)")
    for t, nm in ((attention_out, "attention_out"), (dout, "dout")):
        if tuple(t.shape) != (t1, n1, d2):
            raise ValueError(f"{nm} must be (T1, N1, D2)")
    for t, nm in ((softmax_max, "softmax_max"), (softmax_sum, "softmax_sum")):
        _out(t, (t1, n1, 8), torch.float32, dev, nm)
    _same_device(q, (kcmp, "kcmp"), (vcmp, "vcmp"), (attention_out, "attention_out"), (dout, "dout"))
    cq, cc = _cu(cu_seqlens_q), _cu(cu_cmp_kv)
    if cq.size != cc.size:
        raise ValueError("the prefix-sum lists need one entry per sequence")
    if int(cq[-1]) > t1 or int(cc[-1]) > tc:
        raise ValueError("prefix sums run past the rows of q / kcmp")
    if grads is None:
        dq = _empty(t1, n1, d1, dtype=torch.float32, device=dev)
        dk = _empty(tc, n2, d1, dtype=torch.float32, device=dev)
        dv = _empty(tc, n2, d2, dtype=torch.float32, device=dev)
    else:
        dq, dk, dv = grads
        _out(dq, (t1, n1, d1), torch.float32, dev, "dq")
        _out(dk, (tc, n2, d1), torch.float32, dev, "dkcmp")
        _out(dv, (tc, n2, d2), torch.float32, dev, "dvcmp")
    nbytes = nsa_compress_attention_backward_workspace_size(n1, n2, d1, d2, l, d, cq, cc)
    workspace = _workspace(workspace, nbytes, dev)
    st = load().nsa_compress_attention_backward(
        q.data_ptr(), kcmp.data_ptr(), vcmp.data_ptr(), attention_out.data_ptr(), dout.data_ptr(),
        softmax_max.data_ptr(), softmax_sum.data_ptr(), float(scale), n1, int(l), int(d), _ip(cq), _ip(cc),
        cq.size, n2, d1, d2, dt, dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
        workspace.numel(), _stream(stream))
    _raise(st, "nsa_compress_attention_backward", guards=True)
    return dq, dk, dv


def nsa_compress_backward_workspace_size(cu_seqlens, l: int, d: int) -> int:
    cu = _cu(cu_seqlens)
    out = ctypes.c_size_t(0)
    _raise(load().nsa_compress_backward_workspace_size(_ip(cu), cu.size, int(l), int(d), ctypes.byref(out)),
           "nsa_compress_backward_workspace_size")
    return int(out.value)


def nsa_compress_backward(k: torch.Tensor, v: Optional[torch.Tensor], w: torch.Tensor, dkcmp: torch.Tensor,
                          dvcmp: Optional[torch.Tensor], l: int, d: int, cu_seqlens, grads=None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """Gradient of nsa_compress: returns (dk (T2,N2,D1), dv (T2,N2,D2) or None,
    dw (l,N2)), fp32, for the incoming fp32 dkcmp / dvcmp."""
    _dev(k, "k")
    _dev(w, "w")
    _dev(dkcmp, "dkcmp")
    dt = _dtype_code(k)
    if w.dtype != k.dtype or (v is not None and v.dtype != k.dtype):
        raise TypeError("k, v and w must share one dtype")
    if (v is None) != (dvcmp is None):
        raise ValueError("v and dvcmp go together")
    t2, n2, d1 = k.shape
    d2 = 0
    cu = _cu(cu_seqlens)
    tc = int(nsa_compress_out_len(cu, l, d)[-1])
    _out(dkcmp, (tc, n2, d1), torch.float32, k.device, "dkcmp")
    if v is not None:
        _dev(v, "v")
        d2 = v.shape[2]
        if tuple(v.shape[:2]) != (t2, n2):
            raise ValueError("v must be (T2, N2, D2) with the T2, N2 of k")
        _out(dvcmp, (tc, n2, d2), torch.float32, k.device, "dvcmp")
    if tuple(w.shape) != (l, n2):
        raise ValueError("w must have shape (l, N2)")
    if int(cu[-1]) > t2:
        raise ValueError("cu_seqlens runs past the rows of k")
    _same_device(k, (w, "w"), (v, "v"), (dkcmp, "dkcmp"), (dvcmp, "dvcmp"))
    dev = k.device
    if grads is None:
        dk = _zeros(t2, n2, d1, dtype=torch.float32, device=dev)
        dv = _zeros(t2, n2, d2, dtype=torch.float32, device=dev) if v is not None else None
        dw = _empty(l, n2, dtype=torch.float32, device=dev)
    else:
        dk, dv, dw = grads
        _out(dk, (t2, n2, d1), torch.float32, dev, "dk")
        if v is not None:
            _out(dv, (t2, n2, d2), torch.float32, dev, "dv")
        _out(dw, (l, n2), torch.float32, dev, "dw")
    nbytes = nsa_compress_backward_workspace_size(cu, l, d)
    workspace = _workspace(workspace, nbytes, dev)
    st = load().nsa_compress_backward(
        k.data_ptr(), v.data_ptr() if v is not None else None, w.data_ptr(), dkcmp.data_ptr(),
        dvcmp.data_ptr() if v is not None else None, int(l), int(d), _ip(cu), cu.size, n2, d1, d2, dt,
        dk.data_ptr(), dv.data_ptr() if v is not None else None, dw.data_ptr(), workspace.data_ptr(),
        workspace.numel(), _stream(stream))
    _raise(st, "nsa_compress_backward", guards=True)
    return dk, dv, dw


def nsa_compress_attention_paged(q: torch.Tensor, kcmp_pages: torch.Tensor, vcmp_pages: torch.Tensor,
                                 block_table: torch.Tensor, scale: float, head_num: int, l: int, d: int, lp: int,
                                 count: int, cu_seqlens_q, cu_cmp_kv, cu_sel_kv, out=None,
                                 workspace: Optional[torch.Tensor] = None, stream=None):
    """nsa_compress_attention over a paged compressed K/V cache.

    kcmp_pages (num_pages, page_size, N2, D1), vcmp_pages (num_pages, page_size,
    N2, D2), block_table (batch, max_pages) int32 on the device: sequence b's
    compressed block i is row i % page_size of page block_table[b, i // page_size].
    Returns (attention_out, topk_indices, softmax_max, softmax_sum)."""
    for t, nm in ((q, "q"), (kcmp_pages, "kcmp_pages"), (vcmp_pages, "vcmp_pages"), (block_table, "block_table")):
        _dev(t, nm)
    dt = _dtype_code(q)
    if kcmp_pages.dtype != q.dtype or vcmp_pages.dtype != q.dtype:
        raise TypeError("q and the page pools must share one dtype")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise TypeError("block_table must be a 2-D int32 tensor (batch, max_pages)")
    if q.dim() != 3 or kcmp_pages.dim() != 4 or vcmp_pages.dim() != 4:
        raise ValueError("q must be (T1, N1, D1) and the pools (num_pages, page_size, N2, D)")
    t1, n1, d1 = q.shape
    num_pages, page_size, n2, d1k = kcmp_pages.shape
    d2 = vcmp_pages.shape[3]
    if d1k != d1 or tuple(vcmp_pages.shape[:3]) != (num_pages, page_size, n2):
        raise ValueError("kcmp_pages must be (P, page_size, N2, D1) and vcmp_pages (P, page_size, N2, D2)")
    if int(head_num) != n1:
        raise ValueError("head_num must equal the number of query heads")
    cq, cc, cs = _cu(cu_seqlens_q), _cu(cu_cmp_kv), _cu(cu_sel_kv)
    if not (cq.size == cc.size == cs.size == block_table.shape[0]):
        raise ValueError("one prefix-sum entry and one block-table row per sequence")
    if int(cq[-1]) > t1:
        raise ValueError("cu_seqlens_q runs past the rows of q")
    dev = q.device
    _same_device(q, (kcmp_pages, "kcmp_pages"), (vcmp_pages, "vcmp_pages"), (block_table, "block_table"))
    if out is None:
        att = _empty(t1, n1, d2, dtype=q.dtype, device=dev)
        tk = _empty(t1, n2, count, dtype=torch.int32, device=dev)
        smax = _empty(t1, n1, 8, dtype=torch.float32, device=dev)
        ssum = _empty(t1, n1, 8, dtype=torch.float32, device=dev)
    else:
        att, tk, smax, ssum = out
        _out(att, (t1, n1, d2), q.dtype, dev, "attention_out")
        _out(tk, (t1, n2, count), torch.int32, dev, "topk_indices")
        _out(smax, (t1, n1, 8), torch.float32, dev, "softmax_max")
        _out(ssum, (t1, n1, 8), torch.float32, dev, "softmax_sum")
    ws_bytes = nsa_compress_attention_workspace_size(n1, n2, d1, d2, l, d, lp, count, cq, cc, cs)
    workspace = _workspace(workspace, ws_bytes, dev)
    st = load().nsa_compress_attention_paged(
        q.data_ptr(), kcmp_pages.data_ptr(), vcmp_pages.data_ptr(), int(num_pages), int(page_size),
        block_table.data_ptr(), int(block_table.shape[1]), float(scale), n1, int(l), int(d), int(lp), int(count),
        _ip(cq), _ip(cc), _ip(cs), cq.size, n2, d1, d2, dt, att.data_ptr(), tk.data_ptr(), smax.data_ptr(),
        ssum.data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(stream))
    _raise(st, "nsa_compress_attention_paged", guards=True)
    return att, tk, smax, ssum


def nsa_compress_paged(k: torch.Tensor, v: Optional[torch.Tensor], w: torch.Tensor, l: int, d: int, cu_seqlens,
                       kcmp_pages: torch.Tensor, vcmp_pages: Optional[torch.Tensor], block_table: torch.Tensor,
                       first_block=None, stream=None):
    """Compress windows first_block[b] .. n_cmp_b - 1 of every sequence (all when
    first_block is None) into the paged pools kcmp_pages / vcmp_pages
    (num_pages, page_size, N2, D), in place, through block_table (batch,
    max_pages) int32."""
    for t, nm in ((k, "k"), (w, "w"), (kcmp_pages, "kcmp_pages"), (block_table, "block_table")):
        _dev(t, nm)
    dt = _dtype_code(k)
    if w.dtype != k.dtype or kcmp_pages.dtype != k.dtype or (v is not None and v.dtype != k.dtype):
        raise TypeError("k, v, w and the pools must share one dtype")
    if (v is None) != (vcmp_pages is None):
        raise ValueError("v and vcmp_pages go together")
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise TypeError("block_table must be a 2-D int32 tensor (batch, max_pages)")
    t2, n2, d1 = k.shape
    num_pages, page_size = int(kcmp_pages.shape[0]), int(kcmp_pages.shape[1])
    if tuple(kcmp_pages.shape[2:]) != (n2, d1):
        raise ValueError("kcmp_pages must be (num_pages, page_size, N2, D1)")
    d2 = d1
    if v is not None:
        _dev(v, "v")
        _dev(vcmp_pages, "vcmp_pages")
        d2 = v.shape[2]
        if tuple(vcmp_pages.shape) != (num_pages, page_size, n2, d2):
            raise ValueError("vcmp_pages must be (num_pages, page_size, N2, D2)")
    cu = _cu(cu_seqlens)
    if int(cu[-1]) > t2 or block_table.shape[0] != cu.size:
        raise ValueError("cu_seqlens runs past k, or the block table has the wrong number of rows")
    fb = None if first_block is None else _cu(first_block)
    _same_device(k, (w, "w"), (v, "v"), (kcmp_pages, "kcmp_pages"), (vcmp_pages, "vcmp_pages"),
                 (block_table, "block_table"))
    st = load().nsa_compress_paged(
        k.data_ptr(), v.data_ptr() if v is not None else None, w.data_ptr(), int(l), int(d), _ip(cu), cu.size, n2,
        d1, d2, dt, kcmp_pages.data_ptr(), vcmp_pages.data_ptr() if v is not None else None, num_pages, page_size,
        block_table.data_ptr(), int(block_table.shape[1]), _ip(fb) if fb is not None else None, _stream(stream))
    _raise(st, "nsa_compress_paged", guards=True)
    return kcmp_pages, vcmp_pages
