"""Python binding of libqgemm.so, the B200 (sm_100a) quantized linear layer.

Argument marshalling only: every function here passes device pointers, sizes and
the current CUDA stream of its tensors to the C function of the same name in
include/qgemm.h and raises QgError on a non-OK status.  All compute runs in the
library's CUDA kernels; there is no CPU path.  The library must have been built
(``python -m bit_quantized_gemm_group_b200.build``); importing without it raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqgemm.so")

STATUS = {0: "QG_OK", 1: "QG_ERR_NULL", 2: "QG_ERR_SHAPE", 3: "QG_ERR_ALIGN", 4: "QG_ERR_DTYPE",
          5: "QG_ERR_NONFINITE", 6: "QG_ERR_RANGE", 7: "QG_ERR_TIMEOUT", 8: "QG_ERR_CUDA", 9: "QG_ERR_UNSUPPORTED",
          10: "QG_ERR_WORKSPACE"}
QG_OK, QG_ERR_NULL, QG_ERR_SHAPE, QG_ERR_ALIGN, QG_ERR_DTYPE = 0, 1, 2, 3, 4
QG_ERR_NONFINITE, QG_ERR_RANGE, QG_ERR_TIMEOUT, QG_ERR_CUDA, QG_ERR_UNSUPPORTED = 5, 6, 7, 8, 9
QG_ERR_WORKSPACE = 10
QG_F16, QG_BF16 = 0, 1
QG_OP_GEMM_W4A16, QG_OP_GEMM_W8A8, QG_OP_GEMM_W4A8, QG_OP_AWQ_SEARCH, QG_OP_GPTQ = 0, 1, 2, 3, 4

EXPORTS = ["qg_quantize_w4_group", "qg_pack_nibbles", "qg_gemm_w4a16", "qg_smooth_quant_act_i8", "qg_gemm_w8a8",
           "qg_gemm_w4a8", "qg_smooth_scales", "qg_quantize_w8_channel", "qg_device_status", "qg_status_string",
           "qg_last_error", "qg_selftest_bounded_wait", "qg_workspace_size", "qg_gemm_w4a16_noalloc",
           "qg_awq_act_mean", "qg_awq_scales", "qg_awq_scale_act", "qg_awq_search", "qg_outlier_split_w4",
           "qg_outlier_side_add", "qg_gemm_w4a16_outlier", "qg_prune24", "qg_pack24_vals", "qg_gemm_w4a16_24",
           "qg_gptq", "qg_gptq_blocked", "qg_pack24_tc", "qg_gemm_w4a16_24_tc"]


class QgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if status in (QG_ERR_CUDA, QG_ERR_WORKSPACE, QG_ERR_UNSUPPORTED) and _lib is not None:
            msg += " (" + _lib.qg_last_error().decode() + ")"
        super().__init__(msg)


_P, _I, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "qg_quantize_w4_group": [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P],
    "qg_pack_nibbles": [_P, _I, _I, _P, _P],
    "qg_gemm_w4a16": [_P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _SZ, _P],
    "qg_gemm_w4a16_noalloc": [_P, _I, _I, _I, _I, _P, _P, _P, _I, _P, _P],
    "qg_smooth_quant_act_i8": [_P, _I, _I, _P, _P, _P, _P],
    "qg_gemm_w8a8": [_P, _P, _I, _I, _P, _P, _I, _P, _P, _P, _SZ, _P],
    "qg_gemm_w4a8": [_P, _P, _I, _I, _P, _P, _I, _I, _P, _P, _P, _SZ, _P],
    "qg_smooth_scales": [_P, _I, _P, _I, _I, ctypes.c_float, _P, _P, _P],
    "qg_quantize_w8_channel": [_P, _P, _I, _I, _P, _P, _P],
    "qg_outlier_split_w4": [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P],
    "qg_outlier_side_add": [_P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P],
    "qg_gemm_w4a16_outlier": [_P, _I, _I, _I, _I, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "qg_gptq": [_P, _I, _I, _P, _I, _I, ctypes.c_double, _P, _P, _P, _P, _SZ, _P],
    "qg_gptq_blocked": [_P, _I, _I, _P, _I, _I, ctypes.c_double, _P, _P, _P, _P, _SZ, _P],
    "qg_pack24_tc": [_P, _I, _I, _P, _P],
    "qg_gemm_w4a16_24_tc": [_P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P, _SZ, _P],
    "qg_prune24": [_P, _I, _I, _P, _P, _P],
    "qg_pack24_vals": [_P, _P, _I, _I, _P, _P],
    "qg_gemm_w4a16_24": [_P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _P],
    "qg_awq_act_mean": [_P, _I, _I, _P, _P],
    "qg_awq_scales": [_P, _I, ctypes.c_double, _P, _P, _P],
    "qg_awq_scale_act": [_P, _I, _I, _P, _P, _P],
    "qg_awq_search": [_P, _I, _I, _P, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P],
    "qg_device_status": [_P],
    "qg_selftest_bounded_wait": [ctypes.c_uint64, _P],
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libqgemm.so not built at {path}; run python -m bit_quantized_gemm_group_b200.build")
    L = ctypes.CDLL(path)
    for name, argtypes in _SIGS.items():
        f = getattr(L, name)
        f.argtypes = argtypes
        f.restype = ctypes.c_int
    L.qg_status_string.argtypes = [ctypes.c_int]
    L.qg_status_string.restype = ctypes.c_char_p
    L.qg_last_error.argtypes = []
    L.qg_last_error.restype = ctypes.c_char_p
    L.qg_workspace_size.argtypes = [_I, _I, _I, _I]
    L.qg_workspace_size.restype = ctypes.c_size_t
    return L


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libqgemm.so (loaded on first use; raises ImportError if it was never built)."""
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libqgemm takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous (row-major)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str):
    if st != QG_OK:
        raise QgError(st, where)


def qg_quantize_w4_group(W, s_smooth, group, symmetric, codes, scales, zeros, stream=None):
    K, N = W.shape
    _check(lib().qg_quantize_w4_group(_ptr(W), _ptr(s_smooth), K, N, group, int(bool(symmetric)), _ptr(codes),
                                     _ptr(scales), _ptr(zeros), _stream(stream)), "qg_quantize_w4_group")


def qg_pack_nibbles(codes, packed, stream=None):
    K, N = codes.shape
    _check(lib().qg_pack_nibbles(_ptr(codes), K, N, _ptr(packed), _stream(stream)), "qg_pack_nibbles")


_WS = {}


def qg_workspace_size(op: int, M: int, K: int, N: int) -> int:
    return lib().qg_workspace_size(op, M, K, N)


def default_workspace(op, M, K, N, device):
    """A zero-filled workspace for (op, M, K, N), cached per device and grown on demand.
    Calls that may run concurrently (different streams) need workspaces of their own."""
    need = lib().qg_workspace_size(op, M, K, N)
    if need == 0:
        return None
    key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    buf = _WS.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.zeros(max(need, 1 << 20), dtype=torch.uint8, device=device)
        _WS[key] = buf
    return buf


def _ws(workspace, op, M, K, N, device):
    """workspace='auto' -> cached zero-filled buffer; None / False -> no workspace."""
    if isinstance(workspace, str) and workspace == "auto":
        workspace = default_workspace(op, M, K, N, device)
    if workspace is None or workspace is False:
        return None, 0
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def qg_gemm_w4a16(X, packed, scales, zeros, Y, group=128, workspace="auto", stream=None):
    M, K = X.shape
    N = packed.shape[1]
    xdt = QG_BF16 if X.dtype == torch.bfloat16 else QG_F16 if X.dtype == torch.float16 else -1
    wp, wb = _ws(workspace, QG_OP_GEMM_W4A16, M, K, N, X.device)
    _check(lib().qg_gemm_w4a16(_ptr(X), xdt, M, K, N, _ptr(packed), _ptr(scales), _ptr(zeros), group, _ptr(Y), wp, wb,
                              _stream(stream)), "qg_gemm_w4a16")


def qg_gemm_w4a16_noalloc(X, packed, scales, zeros, Y, group=128, stream=None):
    """W4A16 GEMM with no workspace and no allocation (scratch in a static device array)."""
    M, K = X.shape
    N = packed.shape[1]
    xdt = QG_BF16 if X.dtype == torch.bfloat16 else QG_F16 if X.dtype == torch.float16 else -1
    _check(lib().qg_gemm_w4a16_noalloc(_ptr(X), xdt, M, K, N, _ptr(packed), _ptr(scales), _ptr(zeros), group, _ptr(Y),
                                      _stream(stream)), "qg_gemm_w4a16_noalloc")


def qg_smooth_quant_act_i8(X, inv_s, Xq, t, stream=None):
    M, K = X.shape
    _check(lib().qg_smooth_quant_act_i8(_ptr(X), M, K, _ptr(inv_s), _ptr(Xq), _ptr(t), _stream(stream)),
           "qg_smooth_quant_act_i8")


def qg_gemm_w8a8(Xq, t, Wq, sw, Y, acc_dbg=None, workspace="auto", stream=None):
    M, K = Xq.shape
    N = Wq.shape[1]
    wp, wb = _ws(workspace, QG_OP_GEMM_W8A8, M, K, N, Xq.device)
    _check(lib().qg_gemm_w8a8(_ptr(Xq), _ptr(t), M, K, _ptr(Wq), _ptr(sw), N, _ptr(Y), _ptr(acc_dbg), wp, wb,
                             _stream(stream)), "qg_gemm_w8a8")


def qg_gemm_w4a8(Xq, t, packed, sg, Y, part_dbg=None, group=128, workspace="auto", stream=None):
    M, K = Xq.shape
    N = packed.shape[1]
    wp, wb = _ws(workspace, QG_OP_GEMM_W4A8, M, K, N, Xq.device)
    _check(lib().qg_gemm_w4a8(_ptr(Xq), _ptr(t), M, K, _ptr(packed), _ptr(sg), N, group, _ptr(Y), _ptr(part_dbg), wp,
                             wb, _stream(stream)), "qg_gemm_w4a8")


def qg_smooth_scales(Xcal, W, alpha, s, inv_s, stream=None):
    Mc, K = Xcal.shape
    N = W.shape[1]
    _check(lib().qg_smooth_scales(_ptr(Xcal), Mc, _ptr(W), K, N, ctypes.c_float(alpha), _ptr(s), _ptr(inv_s),
                                 _stream(stream)), "qg_smooth_scales")


def qg_quantize_w8_channel(W, s, Wq, sw, stream=None):
    K, N = W.shape
    _check(lib().qg_quantize_w8_channel(_ptr(W), _ptr(s), K, N, _ptr(Wq), _ptr(sw), _stream(stream)),
           "qg_quantize_w8_channel")


def _xdt(X):
    return QG_BF16 if X.dtype == torch.bfloat16 else QG_F16 if X.dtype == torch.float16 else -1


def qg_outlier_split_w4(W, s_smooth, group, count, idx, codes8, s8, W_dense, stream=None):
    K, N = W.shape
    _check(lib().qg_outlier_split_w4(_ptr(W), _ptr(s_smooth), K, N, group, count, _ptr(idx), _ptr(codes8), _ptr(s8),
                                    _ptr(W_dense), _stream(stream)), "qg_outlier_split_w4")


def qg_outlier_side_add(X, idx, codes8, s8, Y, group=128, stream=None):
    M, K = X.shape
    N = Y.shape[1]
    count = idx.shape[1]
    _check(lib().qg_outlier_side_add(_ptr(X), _xdt(X), M, K, N, group, count, _ptr(idx), _ptr(codes8), _ptr(s8),
                                    _ptr(Y), _stream(stream)), "qg_outlier_side_add")


def qg_gemm_w4a16_outlier(X, packed, scales, zeros, idx, codes8, s8, Y, group=128, workspace="auto", stream=None):
    M, K = X.shape
    N = packed.shape[1]
    count = idx.shape[1]
    wp, wb = _ws(workspace, QG_OP_GEMM_W4A16, M, K, N, X.device)
    _check(lib().qg_gemm_w4a16_outlier(_ptr(X), _xdt(X), M, K, N, _ptr(packed), _ptr(scales), _ptr(zeros), group,
                                      count, _ptr(idx), _ptr(codes8), _ptr(s8), _ptr(Y), wp, wb, _stream(stream)),
           "qg_gemm_w4a16_outlier")


def qg_gptq(Xcal, W, codes, scales, zeros, group=128, damp=0.01, workspace="auto", stream=None):
    Mc, K = Xcal.shape
    N = W.shape[1]
    wp, wb = _ws(workspace, QG_OP_GPTQ, Mc, K, N, Xcal.device)
    _check(lib().qg_gptq(_ptr(Xcal), Mc, K, _ptr(W), N, group, float(damp), _ptr(codes), _ptr(scales), _ptr(zeros), wp,
                        wb, _stream(stream)), "qg_gptq")


def qg_gptq_blocked(Xcal, W, codes, scales, zeros, group=128, damp=0.01, workspace="auto", stream=None):
    Mc, K = Xcal.shape
    N = W.shape[1]
    wp, wb = _ws(workspace, QG_OP_GPTQ, Mc, K, N, Xcal.device)
    _check(lib().qg_gptq_blocked(_ptr(Xcal), Mc, K, _ptr(W), N, group, float(damp), _ptr(codes), _ptr(scales),
                                _ptr(zeros), wp, wb, _stream(stream)), "qg_gptq_blocked")


def qg_prune24(W, Wp, meta, stream=None):
    K, N = W.shape
    _check(lib().qg_prune24(_ptr(W), K, N, _ptr(Wp), _ptr(meta), _stream(stream)), "qg_prune24")


def qg_pack24_vals(codes, meta, vals, stream=None):
    K, N = codes.shape
    _check(lib().qg_pack24_vals(_ptr(codes), _ptr(meta), K, N, _ptr(vals), _stream(stream)), "qg_pack24_vals")


def qg_gemm_w4a16_24(X, vals, meta, scales, zeros, Y, group=128, stream=None):
    M, K = X.shape
    N = vals.shape[1]
    _check(lib().qg_gemm_w4a16_24(_ptr(X), _xdt(X), M, K, N, _ptr(vals), _ptr(meta), _ptr(scales), _ptr(zeros), group,
                                 _ptr(Y), _stream(stream)), "qg_gemm_w4a16_24")


def qg_pack24_tc(vals, vals_tc, stream=None):
    K16, N = vals.shape
    _check(lib().qg_pack24_tc(_ptr(vals), 16 * K16, N, _ptr(vals_tc), _stream(stream)), "qg_pack24_tc")


def qg_gemm_w4a16_24_tc(X, vals_tc, meta, scales, zeros, Y, group=128, workspace="auto", stream=None):
    M, K = X.shape
    N = vals_tc.shape[1]
    wp, wb = _ws(workspace, QG_OP_GEMM_W4A16, M, K, N, X.device)
    _check(lib().qg_gemm_w4a16_24_tc(_ptr(X), _xdt(X), M, K, N, _ptr(vals_tc), _ptr(meta), _ptr(scales), _ptr(zeros),
                                    group, _ptr(Y), wp, wb, _stream(stream)), "qg_gemm_w4a16_24_tc")


def qg_awq_act_mean(Xcal, xm, stream=None):
    Mc, K = Xcal.shape
    _check(lib().qg_awq_act_mean(_ptr(Xcal), Mc, K, _ptr(xm), _stream(stream)), "qg_awq_act_mean")


def qg_awq_scales(xm, alpha, s, inv_s, stream=None):
    _check(lib().qg_awq_scales(_ptr(xm), xm.numel(), float(alpha), _ptr(s), _ptr(inv_s), _stream(stream)),
           "qg_awq_scales")


def qg_awq_scale_act(X, inv_s, Xs, stream=None):
    M, K = X.shape
    _check(lib().qg_awq_scale_act(_ptr(X), M, K, _ptr(inv_s), _ptr(Xs), _stream(stream)), "qg_awq_scale_act")


def qg_awq_search(Xcal, W, n_grid, mse, best, s, inv_s, group=128, workspace="auto", stream=None):
    Mc, K = Xcal.shape
    N = W.shape[1]
    wp, wb = _ws(workspace, QG_OP_AWQ_SEARCH, Mc, K, N, Xcal.device)
    _check(lib().qg_awq_search(_ptr(Xcal), Mc, K, _ptr(W), N, group, n_grid, _ptr(mse), _ptr(best), _ptr(s),
                              _ptr(inv_s), wp, wb, _stream(stream)), "qg_awq_search")


def qg_device_status(stream=None) -> int:
    return lib().qg_device_status(_stream(stream))


def qg_selftest_bounded_wait(limit_ns: int = 0, stream=None):
    _check(lib().qg_selftest_bounded_wait(limit_ns, _stream(stream)), "qg_selftest_bounded_wait")


def qg_status_string(status: int) -> str:
    return lib().qg_status_string(status).decode()
