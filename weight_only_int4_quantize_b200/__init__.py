"""weight_only_int4_quantize_b200: int4 group-128 weight-only quantization, the
W4A16 linear and AWQ candidate scoring on B200 (sm_100a).

This module is a thin ctypes binding over the C ABI of ``libw4.so``
(include/w4.h): it checks tensor devices and dtypes, allocates outputs with
torch and passes raw pointers and the current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback, and
any call fails loudly if the library has not been built
(``python -m weight_only_int4_quantize_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "W4Error", "lib", "quantize_pack", "quantize_pack_batched", "quantize_pack_rows",
    "awq_clip_search_rows", "clip_rows_workspace_bytes", "w4a16_linear",
    "quantize_act_int8", "w4a8_linear", "w4a8_linear_batched", "a8_items",
    "w4a16_linear_batched", "prefill_plan", "awq_scales", "awq_score_grid", "awq_score_grid_static_scratch",
    "awq_workspace_bytes", "device_error", "selftest_bounded_wait",
    "LINEAR_FORCE_GEMV", "LINEAR_FORCE_GEMM", "LINEAR_PDL", "LINEAR_STATIC_WEIGHTS",
    "LINEAR_DECODE_STREAM", "LINEAR_DECODE_TILED", "STREAM_BATCH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4.so")

LINEAR_FORCE_GEMV = 0x1
LINEAR_FORCE_GEMM = 0x2
LINEAR_PDL = 0x4
LINEAR_STATIC_WEIGHTS = 0x8
LINEAR_DECODE_STREAM = 0x10   # decode through the persistent streaming kernel (M <= 8)
LINEAR_DECODE_TILED = 0x20    # decode through the per-CTA tensor-map kernel (M <= 64)
# Linears per launch of w4a16_linear_batched at M <= 8 (one persistent
# streaming launch per this many).
STREAM_BATCH = 256

_STATUS = {
    0: "W4_OK", 1: "W4_ERR_INVALID_ARG", 2: "W4_ERR_SHAPE", 3: "W4_ERR_ALIGNMENT",
    4: "W4_ERR_UNSUPPORTED", 5: "W4_ERR_WORKSPACE", 6: "W4_ERR_CUDA", 7: "W4_ERR_DEVICE_TIMEOUT",
}


class W4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = _STATUS.get(status, str(status))
        msg = lib().w4_status_string(status).decode() if _LIB is not None else self.name
        if status == 6 and _LIB is not None:
            msg += "; " + lib().w4_last_error().decode()
        super().__init__(f"{where}: {self.name} ({msg})")


_LIB: Optional[ctypes.CDLL] = None

_c = ctypes
_p = ctypes.c_void_p
_i64 = ctypes.c_int64


def _declare(L: ctypes.CDLL) -> None:
    L.w4_status_string.restype = ctypes.c_char_p
    L.w4_status_string.argtypes = [ctypes.c_int]
    L.w4_last_error.restype = ctypes.c_char_p
    L.w4_last_error.argtypes = []
    L.w4_abi_version.restype = ctypes.c_int
    L.w4_abi_version.argtypes = []
    L.w4_quantize_pack.restype = ctypes.c_int
    L.w4_quantize_pack.argtypes = [_p, _i64, _i64, ctypes.c_int, ctypes.c_int, _p, ctypes.c_float,
                                   _p, _p, _p, _p]
    L.w4a16_linear.restype = ctypes.c_int
    L.w4a16_linear.argtypes = [_p, _i64, _p, _p, _p, _i64, _i64, ctypes.c_int, _p,
                               ctypes.c_uint, _p]
    L.w4_quantize_pack_batched.restype = ctypes.c_int
    L.w4_quantize_pack_batched.argtypes = [_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p]
    L.w4a16_linear_batched.restype = ctypes.c_int
    L.w4a16_linear_batched.argtypes = [_p, ctypes.c_int, _i64, ctypes.c_int, ctypes.c_uint, _p]
    L.w4_prefill_plan.restype = ctypes.c_int
    L.w4_prefill_plan.argtypes = [_p, _p, ctypes.c_int, _i64, _p, _p, _p, _p]
    L.w4_awq_scales.restype = ctypes.c_int
    L.w4_awq_scales.argtypes = [_p, _i64, _i64, _p, ctypes.c_int, _p, _p]
    L.w4_awq_workspace_bytes.restype = ctypes.c_size_t
    L.w4_awq_workspace_bytes.argtypes = [_i64, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int]
    L.awq_score_grid.restype = ctypes.c_int
    L.awq_score_grid.argtypes = [_p, _i64, _p, _i64, _i64, ctypes.c_int, ctypes.c_int, _p,
                                 ctypes.c_int, _p, ctypes.c_int, _p, ctypes.c_int, _p, _p, _p,
                                 ctypes.c_size_t, _p]
    L.awq_score_grid_static_scratch.restype = ctypes.c_int
    L.awq_score_grid_static_scratch.argtypes = [_p, _i64, _p, _i64, _i64, ctypes.c_int,
                                                ctypes.c_int, _p, ctypes.c_int, _p, ctypes.c_int,
                                                _p, ctypes.c_int, _p, _p, _p]
    L.w4_clip_rows_workspace_bytes.restype = ctypes.c_size_t
    L.w4_clip_rows_workspace_bytes.argtypes = [_i64, _i64, _i64, ctypes.c_int]
    L.awq_clip_search_rows.restype = ctypes.c_int
    L.awq_clip_search_rows.argtypes = [_p, _i64, _p, _i64, _i64, ctypes.c_int, ctypes.c_int, _p,
                                       _p, ctypes.c_int, _p, _p, _p, _p, ctypes.c_size_t, _p]
    L.w4_quantize_pack_rows.restype = ctypes.c_int
    L.w4_quantize_pack_rows.argtypes = [_p, _i64, _i64, ctypes.c_int, ctypes.c_int, _p, _p, _p,
                                        _p, _p, _p]
    L.w4_quantize_act_int8.restype = ctypes.c_int
    L.w4_quantize_act_int8.argtypes = [_p, _i64, _i64, _p, _p, _p, _p]
    L.w4a8_linear.restype = ctypes.c_int
    L.w4a8_linear.argtypes = [_p, _p, _p, _i64, _p, _p, _p, _i64, _i64, ctypes.c_int, _p,
                              ctypes.c_uint, _p]
    L.w4a8_linear_batched.restype = ctypes.c_int
    L.w4a8_linear_batched.argtypes = [_p, ctypes.c_int, _i64, ctypes.c_int, ctypes.c_uint, _p]
    L.w4_block_workspace_bytes.restype = ctypes.c_size_t
    L.w4_block_workspace_bytes.argtypes = [_p, _i64]
    L.awq_block_scoring_losses.restype = ctypes.c_int
    L.awq_block_scoring_losses.argtypes = [_p, _p, _i64, _p, _p, ctypes.c_int, _p, ctypes.c_int,
                                           _p, ctypes.c_int, ctypes.c_int, ctypes.c_int, _p, _p,
                                           ctypes.c_size_t, _p]
    L.awq_block_search.restype = ctypes.c_int
    L.awq_block_search.argtypes = [_p, _p, _i64, _p, _p, _p, ctypes.c_int, _p, ctypes.c_int,
                                   ctypes.c_int, _p, _p, _p, ctypes.c_size_t, _p]
    L.w4_device_error.restype = ctypes.c_int
    L.w4_device_error.argtypes = [ctypes.c_int, _p]
    L.w4_selftest_bounded_wait.restype = ctypes.c_int
    L.w4_selftest_bounded_wait.argtypes = [ctypes.c_uint64, _p]


def lib() -> ctypes.CDLL:
    """The loaded libw4.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m weight_only_int4_quantize_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _LIB = L
    return _LIB


def _check(status: int, where: str) -> None:
    if status != 0:
        raise W4Error(status, where)


def _torch():
    import torch
    return torch


def _stream(device) -> int:
    torch = _torch()
    return torch.cuda.current_stream(device).cuda_stream


def _same_device(ref, **tensors):
    """The kernels run on ref's device and write through every pointer they
    get: all tensors of a call must live on that device."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, the call runs on {ref.device}")


def _cuda(t, dtype, name):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _expect(t, shape, name):
    """Shape check of a companion tensor: the C ABI takes bare pointers and
    cannot see a mis-sized buffer, so the binding refuses it here."""
    if t is not None and tuple(t.shape) != tuple(int(v) for v in shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def quantize_pack(w, symmetric: bool, awq_s=None, shrink: float = 1.0, group: int = 128):
    """RTN int4 g128 quantize+pack of a bf16 [N, K] weight on its device.

    Returns (qweight int32 [N, K/8], scales fp16-bits int16 [N, K/128],
    zeros fp16-bits int16 [N, K/128] or None when symmetric)."""
    torch = _torch()
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    if awq_s is not None:
        _cuda(awq_s, torch.float32, "awq_s")
        _expect(awq_s, (k,), "awq_s")
    qw = torch.empty((n, k // 8), dtype=torch.int32, device=w.device)
    sc = torch.empty((n, k // group), dtype=torch.int16, device=w.device)
    zr = None if symmetric else torch.empty((n, k // group), dtype=torch.int16, device=w.device)
    with torch.cuda.device(w.device):
        st = lib().w4_quantize_pack(w.data_ptr(), n, k, group, int(bool(symmetric)),
                                    None if awq_s is None else awq_s.data_ptr(),
                                    float(shrink), qw.data_ptr(), sc.data_ptr(),
                                    None if zr is None else zr.data_ptr(), _stream(w.device))
    _check(st, "w4_quantize_pack")
    return qw, sc, zr


def quantize_pack_rows(w, symmetric: bool, shrink_rows, awq_s=None, group: int = 128):
    """quantize_pack with one shrink ratio per output row (float32 [N] on the
    weight's device), as chosen by awq_clip_search_rows."""
    torch = _torch()
    _cuda(w, torch.bfloat16, "w")
    _cuda(shrink_rows, torch.float32, "shrink_rows")
    n, k = w.shape
    if shrink_rows.numel() != n:
        raise ValueError("shrink_rows needs one ratio per output row")
    if awq_s is not None:
        _cuda(awq_s, torch.float32, "awq_s")
        _expect(awq_s, (k,), "awq_s")
    qw = torch.empty((n, k // 8), dtype=torch.int32, device=w.device)
    sc = torch.empty((n, k // group), dtype=torch.int16, device=w.device)
    zr = None if symmetric else torch.empty((n, k // group), dtype=torch.int16, device=w.device)
    with torch.cuda.device(w.device):
        st = lib().w4_quantize_pack_rows(w.data_ptr(), n, k, group, int(bool(symmetric)),
                                         None if awq_s is None else awq_s.data_ptr(),
                                         shrink_rows.data_ptr(), qw.data_ptr(), sc.data_ptr(),
                                         None if zr is None else zr.data_ptr(), _stream(w.device))
    _check(st, "w4_quantize_pack_rows")
    return qw, sc, zr


def w4a16_linear(x, qweight, scales, zeros=None, flags: int = 0, group: int = 128, out=None):
    """y = x . dequant(Wq)^T, bf16 [M, K] -> bf16 [M, N]."""
    torch = _torch()
    _cuda(x, torch.bfloat16, "x")
    _cuda(qweight, torch.int32, "qweight")
    _cuda(scales, torch.int16, "scales")
    if zeros is not None:
        _cuda(zeros, torch.int16, "zeros")
    m, k = x.shape
    n = qweight.shape[0]
    if qweight.shape[1] * 8 != k:
        raise ValueError("qweight does not match x's K")
    _expect(scales, (n, k // group), "scales")
    _expect(zeros, (n, k // group), "zeros")
    if out is not None:
        _cuda(out, torch.bfloat16, "out")
        _expect(out, (m, n), "out")
    y = out if out is not None else torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().w4a16_linear(x.data_ptr(), m, qweight.data_ptr(), scales.data_ptr(),
                                None if zeros is None else zeros.data_ptr(), n, k, group,
                                y.data_ptr(), int(flags), _stream(x.device))
    _check(st, "w4a16_linear")
    return y


class QuantItem(ctypes.Structure):
    _fields_ = [("w_bf16", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("awq_s", ctypes.c_void_p), ("shrink", ctypes.c_float),
                ("qweight", ctypes.c_void_p), ("scales_f16", ctypes.c_void_p),
                ("zeros_f16", ctypes.c_void_p)]


class LinearItem(ctypes.Structure):
    _fields_ = [("x_bf16", ctypes.c_void_p), ("qweight", ctypes.c_void_p),
                ("scales_f16", ctypes.c_void_p), ("zeros_f16", ctypes.c_void_p),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("y_bf16", ctypes.c_void_p)]


def quantize_pack_items(items):
    """ctypes array of QuantItem for w4_quantize_pack_batched from
    (w, awq_s or None, shrink, qweight, scales, zeros or None) tuples."""
    arr = (QuantItem * len(items))()
    for a, (w, s, r, qw, sc, zr) in zip(arr, items):
        n, k = w.shape
        _expect(s, (k,), "awq_s")
        _expect(qw, (n, k // 8), "qweight")
        _expect(sc, (n, k // 128), "scales")
        _expect(zr, (n, k // 128), "zeros")
        a.w_bf16, a.N, a.K = w.data_ptr(), w.shape[0], w.shape[1]
        a.awq_s = None if s is None else s.data_ptr()
        a.shrink = float(r)
        a.qweight, a.scales_f16 = qw.data_ptr(), sc.data_ptr()
        a.zeros_f16 = None if zr is None else zr.data_ptr()
    return arr


def quantize_pack_batched(items, symmetric: bool, group: int = 128, stream=None) -> None:
    """Quantize+pack many tensors in few launches; items are tuples
    (w, awq_s or None, shrink, qweight, scales, zeros or None) of CUDA tensors
    (outputs preallocated), or a prepared quantize_pack_items() array."""
    torch = _torch()
    arr = items if isinstance(items, ctypes.Array) else quantize_pack_items(items)
    st = lib().w4_quantize_pack_batched(ctypes.addressof(arr), len(arr), group,
                                        int(bool(symmetric)),
                                        stream if stream is not None else _stream(torch.cuda.current_device()))
    _check(st, "w4_quantize_pack_batched")


def linear_items(items, m=None):
    """ctypes array of LinearItem from (x, qweight, scales, zeros or None, y)
    tuples (x [M, K], y [M, N]; with m given, M must equal it)."""
    arr = (LinearItem * len(items))()
    for a, (x, qw, sc, zr, y) in zip(arr, items):
        mm, k = x.shape
        n = qw.shape[0]
        if m is not None and mm != m:
            raise ValueError(f"x has {mm} rows, the call has {m}")
        _expect(qw, (n, k // 8), "qweight")
        _expect(sc, (n, k // 128), "scales")
        _expect(zr, (n, k // 128), "zeros")
        _expect(y, (mm, n), "y")
        a.x_bf16, a.qweight, a.scales_f16 = x.data_ptr(), qw.data_ptr(), sc.data_ptr()
        a.zeros_f16 = None if zr is None else zr.data_ptr()
        a.N, a.K, a.y_bf16 = qw.shape[0], x.shape[1], y.data_ptr()
    return arr


def prefill_plan(shapes, m: int, resident=None):
    """(tile_rows, tile_cols, k_split) of the prefill launch for linears of
    shapes [(N, K), ...] (at most 16) sharing m rows.  resident: None (the
    current device's counts) or 4 x 4 ints, the CTAs run at once per tile
    shape (256x256, 128x256, 256x128, 128x128) and cluster size 1..4."""
    n = len(shapes)
    na = (ctypes.c_int64 * max(n, 1))(*[int(s[0]) for s in shapes])
    ka = (ctypes.c_int64 * max(n, 1))(*[int(s[1]) for s in shapes])
    res = None
    if resident is not None:
        flat = [int(v) for row in resident for v in row]
        if len(flat) != 16:
            raise ValueError("resident must be 4 x 4")
        res = (ctypes.c_int * 16)(*flat)
    rows, cols, ks = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().w4_prefill_plan(na, ka, n, int(m), res, ctypes.byref(rows), ctypes.byref(cols),
                                 ctypes.byref(ks)), "w4_prefill_plan")
    return rows.value, cols.value, ks.value


def w4a16_linear_batched(items, m: int, flags: int = 0, group: int = 128, stream=None) -> None:
    """Many independent linears with the same token count m in few launches;
    items are (x, qweight, scales, zeros or None, y) tuples of CUDA tensors or
    a prepared linear_items() array."""
    torch = _torch()
    arr = items if isinstance(items, ctypes.Array) else linear_items(items, m)
    st = lib().w4a16_linear_batched(ctypes.addressof(arr), len(arr), int(m), group, int(flags),
                                    stream if stream is not None else _stream(torch.cuda.current_device()))
    _check(st, "w4a16_linear_batched")


def quantize_act_int8(x):
    """Per-token int8 activations for W4A8: (xq int8 [M, K] in the library's
    chunk channel order, xsum int32 [M, K/128], xscale float32 [M])."""
    torch = _torch()
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    xq = torch.empty((m, k), dtype=torch.int8, device=x.device)
    xs = torch.empty((m, k // 128), dtype=torch.int32, device=x.device)
    sc = torch.empty((m,), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().w4_quantize_act_int8(x.data_ptr(), m, k, xq.data_ptr(), xs.data_ptr(),
                                        sc.data_ptr(), _stream(x.device))
    _check(st, "w4_quantize_act_int8")
    return xq, xs, sc


def w4a8_linear(xq, xsum, xscale, qweight, scales, zeros=None, flags: int = 0, group: int = 128,
                out=None):
    """y = W4A8 decode of int8 activations (from quantize_act_int8), bf16 [M, N]."""
    torch = _torch()
    _cuda(xq, torch.int8, "xq")
    _cuda(xsum, torch.int32, "xsum")
    _cuda(xscale, torch.float32, "xscale")
    _cuda(qweight, torch.int32, "qweight")
    _cuda(scales, torch.int16, "scales")
    if zeros is not None:
        _cuda(zeros, torch.int16, "zeros")
    m, k = xq.shape
    n = qweight.shape[0]
    _expect(xsum, (m, k // 128), "xsum")
    _expect(xscale, (m,), "xscale")
    _expect(qweight, (n, k // 8), "qweight")
    _expect(scales, (n, k // group), "scales")
    _expect(zeros, (n, k // group), "zeros")
    if out is not None:
        _cuda(out, torch.bfloat16, "out")
        _expect(out, (m, n), "out")
    y = out if out is not None else torch.empty((m, n), dtype=torch.bfloat16, device=xq.device)
    with torch.cuda.device(xq.device):
        st = lib().w4a8_linear(xq.data_ptr(), xsum.data_ptr(), xscale.data_ptr(), m,
                               qweight.data_ptr(), scales.data_ptr(),
                               None if zeros is None else zeros.data_ptr(), n, k, group,
                               y.data_ptr(), int(flags), _stream(xq.device))
    _check(st, "w4a8_linear")
    return y


class A8Item(ctypes.Structure):
    _fields_ = [("xq", ctypes.c_void_p), ("xsum", ctypes.c_void_p), ("xscale", ctypes.c_void_p),
                ("qweight", ctypes.c_void_p), ("scales_f16", ctypes.c_void_p),
                ("zeros_f16", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("y_bf16", ctypes.c_void_p)]


def a8_items(items, m=None):
    """Host array of w4a8_item from (xq, xsum, xscale, qweight, scales, zeros, y) tuples."""
    arr = (A8Item * len(items))()
    for i, (xq, xs, sc_x, qw, sc, zr, y) in enumerate(items):
        mm, k = xq.shape
        n = qw.shape[0]
        if m is not None and mm != m:
            raise ValueError(f"xq has {mm} rows, the call has {m}")
        _expect(xs, (mm, k // 128), "xsum")
        _expect(sc_x, (mm,), "xscale")
        _expect(qw, (n, k // 8), "qweight")
        _expect(sc, (n, k // 128), "scales")
        _expect(zr, (n, k // 128), "zeros")
        _expect(y, (mm, n), "y")
        arr[i] = A8Item(xq.data_ptr(), xs.data_ptr(), sc_x.data_ptr(), qw.data_ptr(),
                        sc.data_ptr(), None if zr is None else zr.data_ptr(), qw.shape[0],
                        xq.shape[1], y.data_ptr())
    return arr


def w4a8_linear_batched(items, m: int, flags: int = 0, group: int = 128, stream=None) -> None:
    """Many independent W4A8 linears with the same token count m."""
    torch = _torch()
    arr = items if isinstance(items, ctypes.Array) else a8_items(items, m)
    st = lib().w4a8_linear_batched(ctypes.addressof(arr), len(arr), int(m), group, int(flags),
                                   stream if stream is not None else _stream(torch.cuda.current_device()))
    _check(st, "w4a8_linear_batched")


def awq_scales(x, alphas: Sequence[float]):
    """s [n_alpha, K] float32 = max(mean|x|, 1e-8) ** alpha per input channel."""
    torch = _torch()
    import numpy as np
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    a = np.ascontiguousarray(np.asarray(alphas, dtype=np.float32))
    s = torch.empty((len(a), k), dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().w4_awq_scales(x.data_ptr(), m, k, a.ctypes.data, len(a), s.data_ptr(),
                                 _stream(x.device))
    _check(st, "w4_awq_scales")
    return s


def awq_workspace_bytes(m: int, n: int, k: int, n_alpha: int, n_shrink: int, n_seg: int = 1) -> int:
    return int(lib().w4_awq_workspace_bytes(m, n, k, n_alpha, n_shrink, n_seg))


def awq_score_grid(x, w, alphas, shrinks, symmetric: bool, seg_offsets=None, workspace=None,
                   group: int = 128):
    """SSE table [n_seg, n_alpha, n_shrink] (float64) and argmins [n_seg+1, 4]
    (int32) of every (alpha, shrink) candidate, on the tensors' device."""
    torch = _torch()
    import numpy as np
    _cuda(x, torch.bfloat16, "x")
    _cuda(w, torch.bfloat16, "w")
    _same_device(x, w=w)
    m, k = x.shape
    n = w.shape[0]
    _expect(w, (n, k), "w")
    a = np.ascontiguousarray(np.asarray(alphas, dtype=np.float32))
    r = np.ascontiguousarray(np.asarray(shrinks, dtype=np.float32))
    if seg_offsets is None:
        seg = None
        n_seg = 1
    else:
        seg = np.ascontiguousarray(np.asarray(seg_offsets, dtype=np.int64))
        n_seg = len(seg) - 1
    need = awq_workspace_bytes(m, n, k, len(a), len(r), n_seg)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    sse = torch.empty((n_seg, len(a), len(r)), dtype=torch.float64, device=x.device)
    arg = torch.empty((n_seg + 1, 4), dtype=torch.int32, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().awq_score_grid(x.data_ptr(), m, w.data_ptr(), n, k, group,
                                  int(bool(symmetric)), a.ctypes.data, len(a), r.ctypes.data,
                                  len(r), None if seg is None else seg.ctypes.data, n_seg,
                                  sse.data_ptr(), arg.data_ptr(), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(),
                                  _stream(x.device))
    _check(st, "awq_score_grid")
    return sse, arg


def clip_rows_workspace_bytes(m: int, n: int, k: int, n_shrink: int) -> int:
    return int(lib().w4_clip_rows_workspace_bytes(m, n, k, n_shrink))


def awq_clip_search_rows(x, w, shrinks, symmetric: bool, awq_s=None, workspace=None,
                         group: int = 128):
    """Per-output-channel clipping search: (sse_rows float64 [n_shrink, N],
    choice int32 [N], shrink_rows float32 [N]) on the tensors' device."""
    torch = _torch()
    import numpy as np
    _cuda(x, torch.bfloat16, "x")
    _cuda(w, torch.bfloat16, "w")
    _same_device(x, w=w)
    if awq_s is not None:
        _cuda(awq_s, torch.float32, "awq_s")
    m, k = x.shape
    n = w.shape[0]
    _expect(w, (n, k), "w")
    _expect(awq_s, (k,), "awq_s")
    r = np.ascontiguousarray(np.asarray(shrinks, dtype=np.float32))
    if workspace is None:
        workspace = torch.empty(clip_rows_workspace_bytes(m, n, k, len(r)), dtype=torch.uint8,
                                device=x.device)
    sse = torch.empty((len(r), n), dtype=torch.float64, device=x.device)
    choice = torch.empty(n, dtype=torch.int32, device=x.device)
    rows = torch.empty(n, dtype=torch.float32, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().awq_clip_search_rows(x.data_ptr(), m, w.data_ptr(), n, k, group,
                                        int(bool(symmetric)),
                                        None if awq_s is None else awq_s.data_ptr(),
                                        r.ctypes.data, len(r), sse.data_ptr(), choice.data_ptr(),
                                        rows.data_ptr(), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(x.device))
    _check(st, "awq_clip_search_rows")
    return sse, choice, rows


def awq_score_grid_static_scratch(x, w, alphas, shrinks, symmetric: bool, seg_offsets=None,
                                  sse_out=None, argmin_out=None, group: int = 128):
    """awq_score_grid with the library's fixed device scratch instead of a
    workspace.  The C call allocates nothing; pass preallocated sse_out
    [n_seg, n_alpha, n_shrink] float64 and argmin_out [n_seg + 1, 4] int32
    to keep this binding from allocating them."""
    torch = _torch()
    import numpy as np
    _cuda(x, torch.bfloat16, "x")
    _cuda(w, torch.bfloat16, "w")
    _same_device(x, w=w)
    m, k = x.shape
    n = w.shape[0]
    _expect(w, (n, k), "w")
    a = np.ascontiguousarray(np.asarray(alphas, dtype=np.float32))
    r = np.ascontiguousarray(np.asarray(shrinks, dtype=np.float32))
    seg = None if seg_offsets is None else np.ascontiguousarray(np.asarray(seg_offsets, dtype=np.int64))
    n_seg = 1 if seg is None else len(seg) - 1
    if sse_out is None:
        sse_out = torch.empty((n_seg, len(a), len(r)), dtype=torch.float64, device=x.device)
    if argmin_out is None:
        argmin_out = torch.empty((n_seg + 1, 4), dtype=torch.int32, device=x.device)
    _cuda(sse_out, torch.float64, "sse_out")
    _cuda(argmin_out, torch.int32, "argmin_out")
    if tuple(sse_out.shape) != (n_seg, len(a), len(r)) or tuple(argmin_out.shape) != (n_seg + 1, 4):
        raise ValueError("sse_out / argmin_out have the wrong shape")
    _same_device(x, w=w, sse_out=sse_out, argmin_out=argmin_out)
    with torch.cuda.device(x.device):
        st = lib().awq_score_grid_static_scratch(
            x.data_ptr(), m, w.data_ptr(), n, k, group, int(bool(symmetric)), a.ctypes.data,
            len(a), r.ctypes.data, len(r), None if seg is None else seg.ctypes.data, n_seg,
            sse_out.data_ptr(), argmin_out.data_ptr(), _stream(x.device))
    if st == 5:  # W4_ERR_WORKSPACE: the problem does not fit the static scratch
        raise W4Error(st, "awq_score_grid_static_scratch: " + lib().w4_last_error().decode())
    _check(st, "awq_score_grid_static_scratch")
    return sse_out, argmin_out


class BlockConfig(ctypes.Structure):
    """w4_block_config: a decoder block's shape (Qwen3 conventions)."""
    _fields_ = [("hidden", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ffn", ctypes.c_int32), ("eps", ctypes.c_double),
                ("rope_theta", ctypes.c_double)]


class _BlockWeights(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("q", "k", "v", "o", "gate", "up", "down", "ln1", "ln2", "q_norm", "k_norm")]


QWEN3_1P7B_BLOCK = dict(hidden=2048, heads=16, kv_heads=8, head_dim=128, ffn=6144, eps=1e-6,
                        rope_theta=1e6)
BLOCK_LINEARS = ("q", "k", "v", "o", "gate", "up", "down")
BLOCK_GROUPS = ("qkv", "o", "gate_up", "down")


def _block_cfg(cfg):
    return BlockConfig(**(cfg or QWEN3_1P7B_BLOCK))


def _block_weights(blk, ref):
    """Checks one block's tensors (dict: the seven bf16 linears, the four
    float64 gains) and returns the C struct of their pointers."""
    if blk is None:
        return None
    torch = _torch()
    for name in BLOCK_LINEARS:
        _cuda(blk[name], torch.bfloat16, name)
    for name in ("ln1", "ln2", "q_norm", "k_norm"):
        _cuda(blk[name], torch.float64, name)
    _same_device(ref, **{k: blk[k] for k in BLOCK_LINEARS + ("ln1", "ln2", "q_norm", "k_norm")})
    return _BlockWeights(**{f[0]: blk[f[0]].data_ptr() for f in _BlockWeights._fields_})


def block_workspace_bytes(t: int, cfg=None) -> int:
    c = _block_cfg(cfg)
    return int(lib().w4_block_workspace_bytes(ctypes.byref(c), int(t)))


def _block_common(x, block, next_block, alphas, shrinks, cfg, workspace):
    import numpy as np
    torch = _torch()
    _cuda(x, torch.float64, "x")
    c = _block_cfg(cfg)
    t = x.shape[0]
    if x.dim() != 2 or x.shape[1] != c.hidden:
        raise ValueError("x must be float64 [T, hidden]")
    bi = _block_weights(block, x)
    bn = _block_weights(next_block, x)
    al = np.ascontiguousarray(np.asarray(alphas, dtype=np.float32))
    sh = np.ascontiguousarray(np.asarray(shrinks, dtype=np.float32))
    need = int(lib().w4_block_workspace_bytes(ctypes.byref(c), t))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    _same_device(x, workspace=workspace)
    return c, t, bi, bn, al, sh, workspace


def awq_block_scoring_losses(x, block, next_block, group, alphas, shrinks, symmetric: bool,
                             only=None, cfg=None, workspace=None):
    """loss[a, j] of every (alphas[a], shrinks[j]) candidate of one linear
    group of a decoder block, at the output of next_block (look-ahead) or of
    the block itself (next_block None), in binary64 on the device.

    x: float64 [T, hidden] block input on the device; block / next_block:
    dicts of the seven bf16 linears ("q" .. "down", [out, in]) and the float64
    gains "ln1", "ln2", "q_norm", "k_norm"; group: "qkv", "o", "gate_up",
    "down" (or 0..3); only: None or the name of one linear of the group."""
    torch = _torch()
    c, t, bi, bn, al, sh, ws = _block_common(x, block, next_block, alphas, shrinks, cfg,
                                             workspace)
    g = BLOCK_GROUPS.index(group) if isinstance(group, str) else int(group)
    o = -1 if only is None else (BLOCK_LINEARS.index(only) if isinstance(only, str) else int(only))
    losses = torch.empty((len(al), len(sh)), dtype=torch.float64, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().awq_block_scoring_losses(
            ctypes.byref(c), x.data_ptr(), t, ctypes.byref(bi),
            None if bn is None else ctypes.byref(bn), g, al.ctypes.data, len(al),
            sh.ctypes.data, len(sh), int(bool(symmetric)), o, losses.data_ptr(),
            ws.data_ptr(), ws.numel(), _stream(x.device))
    _check(st, "awq_block_scoring_losses")
    return losses


def awq_block_search(x, block, next_block, alphas, shrinks, symmetric: bool, cfg=None,
                     workspace=None):
    """The search of one block on the device: returns (choice int32 [11]:
    alpha index per group qkv, o, gate_up, down, then shrink index per
    linear q .. down; losses float64 [4 * n_alpha + 7 * n_shrink])."""
    torch = _torch()
    c, t, bi, bn, al, sh, ws = _block_common(x, block, next_block, alphas, shrinks, cfg,
                                             workspace)
    choice = torch.empty(11, dtype=torch.int32, device=x.device)
    losses = torch.empty(4 * len(al) + 7 * len(sh), dtype=torch.float64, device=x.device)
    with torch.cuda.device(x.device):
        st = lib().awq_block_search(
            ctypes.byref(c), x.data_ptr(), t, ctypes.byref(bi),
            None if bn is None else ctypes.byref(bn), al.ctypes.data, len(al), sh.ctypes.data,
            len(sh), int(bool(symmetric)), choice.data_ptr(), losses.data_ptr(), ws.data_ptr(),
            ws.numel(), _stream(x.device))
    _check(st, "awq_block_search")
    return choice, losses


def device_error(clear: bool = True) -> int:
    """The library's device error word (0 = no kernel gave up on a wait)."""
    code = ctypes.c_uint32(0)
    st = lib().w4_device_error(int(bool(clear)), ctypes.byref(code))
    if st not in (0, 7):
        _check(st, "w4_device_error")
    return int(code.value)


def selftest_bounded_wait(limit_ns: int = 20_000_000) -> None:
    """Launches the bounded-wait self-test kernel on the current stream."""
    torch = _torch()
    _check(lib().w4_selftest_bounded_wait(int(limit_ns), _stream(torch.cuda.current_device())),
           "w4_selftest_bounded_wait")
