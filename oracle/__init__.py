"""CPU oracle for the quantized linear layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  The product library
(``bit_quantized_gemm_group_b200``) never imports it and shares no code with
it: the arithmetic lives in ``qg_oracle.c`` (plain C, binary32 for every stored
integer or scale, binary64 for GEMM references); this module only builds that
file with gcc and marshals numpy arrays into it.

Each wrapper names the passage of the pages its C function follows; the
function comments in ``qg_oracle.c`` give the full statement and the readings
taken where the pages are silent.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force on tiny inputs, special cases that reduce to a
library matmul, invariants).  None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qg_oracle.c")
_LIB = os.path.join(_HERE, "libqg_oracle.so")

OK, NONFINITE, RANGE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile qg_oracle.c into libqg_oracle.so (plain gcc, IEEE semantics kept)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-std=c11",
               "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int


def _declare(L):
    L.qgo_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.qgo_f16_to_f32.restype = ctypes.c_float
    L.qgo_f32_to_f16_ru.argtypes = [ctypes.c_float]
    L.qgo_f32_to_f16_ru.restype = ctypes.c_uint16
    L.qgo_f32_to_bf16_rn.argtypes = [ctypes.c_float]
    L.qgo_f32_to_bf16_rn.restype = ctypes.c_uint16
    L.qgo_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.qgo_bf16_to_f32.restype = ctypes.c_float
    L.qgo_quantize_w4_asym.argtypes = [_p, _p, _i64, _i64, _int, _p, _p, _p]
    L.qgo_quantize_w4_asym.restype = _int
    L.qgo_quantize_w4_sym.argtypes = [_p, _p, _i64, _i64, _int, _p, _p]
    L.qgo_quantize_w4_sym.restype = _int
    L.qgo_pack_nibbles.argtypes = [_p, _i64, _i64, _p]
    L.qgo_pack_nibbles.restype = None
    L.qgo_unpack_nibbles.argtypes = [_p, _i64, _i64, _p]
    L.qgo_unpack_nibbles.restype = None
    L.qgo_gemm_w4a16_ref.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _int, _p, _i64, _p, _p]
    L.qgo_gemm_w4a16_ref.restype = None
    L.qgo_smooth_scales.argtypes = [_p, _i64, _p, _i64, _i64, ctypes.c_float, _p, _p]
    L.qgo_smooth_scales.restype = _int
    L.qgo_smooth_quant_act_i8.argtypes = [_p, _i64, _i64, _p, _p, _p]
    L.qgo_smooth_quant_act_i8.restype = _int
    L.qgo_quantize_w8_channel.argtypes = [_p, _p, _i64, _i64, _p, _p]
    L.qgo_quantize_w8_channel.restype = _int
    L.qgo_gemm_w8a8.argtypes = [_p, _p, _i64, _i64, _p, _p, _i64, _p, _i64, _p, _p, _p, _p]
    L.qgo_gemm_w8a8.restype = None
    L.qgo_gemm_w4a8.argtypes = [_p, _p, _i64, _i64, _p, _p, _i64, _int, _p, _i64, _p, _p, _p, _p]
    L.qgo_gemm_w4a8.restype = None
    L.qgo_gemm_f64.argtypes = [_p, _i64, _i64, _p, _i64, _p, _i64, _p]
    L.qgo_gemm_f64.restype = None
    L.qgo_outlier_count.argtypes = [_int]
    L.qgo_outlier_count.restype = _int
    L.qgo_outlier_split.argtypes = [_p, _p, _i64, _i64, _int, _int, _p, _p, _p, _p]
    L.qgo_outlier_split.restype = _int
    L.qgo_gemm_w4a16_outlier_ref.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _int, _int, _p, _p, _p, _p, _i64,
                                             _p, _p]
    L.qgo_gemm_w4a16_outlier_ref.restype = None
    L.qgo_prune24.argtypes = [_p, _i64, _i64, _p, _p]
    L.qgo_prune24.restype = None
    L.qgo_pack24_vals.argtypes = [_p, _p, _i64, _i64, _p]
    L.qgo_pack24_vals.restype = None
    L.qgo_gemm_w4a16_24_ref.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _p, _int, _p, _i64, _p, _p]
    L.qgo_gemm_w4a16_24_ref.restype = None
    L.qgo_gptq_hessian.argtypes = [_p, _i64, _i64, ctypes.c_double, _p]
    L.qgo_gptq_hessian.restype = None
    L.qgo_gptq.argtypes = [_p, _i64, _i64, _p, _i64, _int, ctypes.c_double, _p, _p, _p]
    L.qgo_gptq.restype = _int
    L.qgo_gptq_replay.argtypes = [_p, _i64, _i64, _p, _i64, _int, ctypes.c_double, _p, _p, _p, _int, _p, _p, _p]
    L.qgo_gptq_replay.restype = _int
    L.qgo_awq_act_mean.argtypes = [_p, _i64, _i64, _p]
    L.qgo_awq_act_mean.restype = None
    L.qgo_awq_scales.argtypes = [_p, _i64, ctypes.c_double, _p, _p]
    L.qgo_awq_scales.restype = None
    L.qgo_awq_scale_act.argtypes = [_p, _i64, _i64, _p, _p]
    L.qgo_awq_scale_act.restype = None
    L.qgo_awq_alpha.argtypes = [_int, _int]
    L.qgo_awq_alpha.restype = ctypes.c_double
    L.qgo_awq_candidate_mse.argtypes = [_p, _i64, _i64, _p, _i64, _int, _p, _p, _p, _p]
    L.qgo_awq_candidate_mse.restype = _int
    L.qgo_awq_search.argtypes = [_p, _i64, _i64, _p, _i64, _int, _int, _p, _p, _p, _p]
    L.qgo_awq_search.restype = _int


def _c(a, dtype):
    """C-contiguous array of the given dtype (no copy if already so)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows):
    if rows is None:
        return None, 0
    r = _c(rows, np.int64)
    return r, r.size


# --------------------------------------------------------------------------
# scalar conversions (IEEE binary16 / bfloat16 definitions)
# --------------------------------------------------------------------------
def f16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = _c(bits, np.uint16).ravel()
    return np.array([lib().qgo_f16_to_f32(int(x)) for x in b], dtype=np.float32).reshape(np.shape(bits))


def f32_to_f16_ru(x: np.ndarray) -> np.ndarray:
    v = _c(x, np.float32).ravel()
    return np.array([lib().qgo_f32_to_f16_ru(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(x))


def f32_to_bf16_rn(x: np.ndarray) -> np.ndarray:
    v = _c(x, np.float32).ravel()
    return np.array([lib().qgo_f32_to_bf16_rn(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(x))


# --------------------------------------------------------------------------
# quantizers  ("AI Infra guide, ch.4 Quantization" sec. 1.1-1.3; SmoothQuant sec. 2.2;
#              "LLM inference cost: W8A8/W4A8 ..." sec. 2.2, group size 128)
# --------------------------------------------------------------------------
def quantize_w4_asym(W, group=128, s_smooth=None):
    """Asymmetric INT4 per group of `group` rows along K -> (codes u8 [K][N],
    scales fp16 bits [K/g][N], zeros u8 [K/g][N], status)."""
    W = _c(W, np.float32)
    K, N = W.shape
    s = None if s_smooth is None else _c(s_smooth, np.float32)
    codes = np.zeros((K, N), np.uint8)
    scales = np.zeros((K // group, N), np.uint16)
    zeros = np.zeros((K // group, N), np.uint8)
    st = lib().qgo_quantize_w4_asym(_ptr(W), _ptr(s), K, N, group, _ptr(codes), _ptr(scales), _ptr(zeros))
    return codes, scales, zeros, st


def quantize_w4_sym(W, group=128, s_smooth=None):
    """Symmetric INT4 (s = max|w|/7, codes in [-7,7]) -> (codes i8 [K][N], scales f32 [K/g][N], status)."""
    W = _c(W, np.float32)
    K, N = W.shape
    s = None if s_smooth is None else _c(s_smooth, np.float32)
    codes = np.zeros((K, N), np.int8)
    scales = np.zeros((K // group, N), np.float32)
    st = lib().qgo_quantize_w4_sym(_ptr(W), _ptr(s), K, N, group, _ptr(codes), _ptr(scales))
    return codes, scales, st


def pack_nibbles(codes):
    """codes [K][N] (u8, or i8 two's complement) -> packed u32 [K/8][N], low nibble first along K."""
    c = _c(np.asarray(codes).view(np.uint8), np.uint8)
    K, N = c.shape
    packed = np.zeros((K // 8, N), np.uint32)
    lib().qgo_pack_nibbles(_ptr(c), K, N, _ptr(packed))
    return packed


def unpack_nibbles(packed, K):
    p = _c(packed, np.uint32)
    N = p.shape[1]
    codes = np.zeros((K, N), np.uint8)
    lib().qgo_unpack_nibbles(_ptr(p), K, N, _ptr(codes))
    return codes


def smooth_scales(Xcal, W, alpha=0.5):
    """SmoothQuant s_j = max|X_j|^a / max|W_j|^(1-a) and inv_s = 1/s -> (s, inv_s, status)."""
    Xc = _c(Xcal, np.float32)
    Wc = _c(W, np.float32)
    Mc, K = Xc.shape
    N = Wc.shape[1]
    s = np.zeros(K, np.float32)
    inv = np.zeros(K, np.float32)
    st = lib().qgo_smooth_scales(_ptr(Xc), Mc, _ptr(Wc), K, N, ctypes.c_float(alpha), _ptr(s), _ptr(inv))
    return s, inv, st


def smooth_quant_act_i8(X, inv_s=None):
    """Per-token symmetric INT8 of X * inv_s -> (Xq i8 [M][K], t f32 [M], status)."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    inv = None if inv_s is None else _c(inv_s, np.float32)
    Xq = np.zeros((M, K), np.int8)
    t = np.zeros(M, np.float32)
    st = lib().qgo_smooth_quant_act_i8(_ptr(Xc), M, K, _ptr(inv), _ptr(Xq), _ptr(t))
    return Xq, t, st


def quantize_w8_channel(W, s_smooth=None):
    """Per-output-channel symmetric INT8 of diag(s) W -> (Wq i8 [K][N], sw f32 [N], status)."""
    Wc = _c(W, np.float32)
    K, N = Wc.shape
    s = None if s_smooth is None else _c(s_smooth, np.float32)
    Wq = np.zeros((K, N), np.int8)
    sw = np.zeros(N, np.float32)
    st = lib().qgo_quantize_w8_channel(_ptr(Wc), _ptr(s), K, N, _ptr(Wq), _ptr(sw))
    return Wq, sw, st


# --------------------------------------------------------------------------
# GEMM references
# --------------------------------------------------------------------------
def gemm_w4a16_ref(X, packed, scales, zeros, group=128, rows=None):
    """fp64 y = X * W_deq and bound = |X| * |W_deq| for the selected rows."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    p = _c(packed, np.uint32)
    N = p.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    y = np.zeros((nr, N), np.float64)
    b = np.zeros((nr, N), np.float64)
    lib().qgo_gemm_w4a16_ref(_ptr(Xc), M, K, N, _ptr(p), _ptr(_c(scales, np.uint16)), _ptr(_c(zeros, np.uint8)),
                             group, _ptr(r), nr, _ptr(y), _ptr(b))
    return y, b


def gemm_w8a8(Xq, t, Wq, sw, rows=None):
    """-> (acc i32, Y bf16 bits, yref f64, bound f64) for the selected rows."""
    Xq = _c(Xq, np.int8)
    M, K = Xq.shape
    Wq = _c(Wq, np.int8)
    N = Wq.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    acc = np.zeros((nr, N), np.int32)
    y = np.zeros((nr, N), np.uint16)
    yref = np.zeros((nr, N), np.float64)
    b = np.zeros((nr, N), np.float64)
    lib().qgo_gemm_w8a8(_ptr(Xq), _ptr(_c(t, np.float32)), M, K, _ptr(Wq), _ptr(_c(sw, np.float32)), N,
                        _ptr(r), nr, _ptr(acc), _ptr(y), _ptr(yref), _ptr(b))
    return acc, y, yref, b


def gemm_w4a8(Xq, t, packed, sg, group=128, rows=None, want_part=True, want_y=False):
    """-> (part i32 [rows][K/g][N] or None, yref f64, bound f64) for the selected rows;
    with want_y also the output bf16 bits as the workload defines it (binary32 group
    products summed in ascending group order, times t, rounded once)."""
    Xq = _c(Xq, np.int8)
    M, K = Xq.shape
    p = _c(packed, np.uint32)
    N = p.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    part = np.zeros((nr, K // group, N), np.int32) if want_part else None
    yref = np.zeros((nr, N), np.float64)
    b = np.zeros((nr, N), np.float64)
    y = np.zeros((nr, N), np.uint16) if want_y else None
    lib().qgo_gemm_w4a8(_ptr(Xq), _ptr(_c(t, np.float32)), M, K, _ptr(p), _ptr(_c(sg, np.float32)), N, group,
                        _ptr(r), nr, _ptr(part), _ptr(yref), _ptr(b), _ptr(y))
    if want_y:
        return part, yref, b, y
    return part, yref, b


def gemm_f64(X, W, rows=None):
    Xc = _c(X, np.float32)
    Wc = _c(W, np.float32)
    M, K = Xc.shape
    N = Wc.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    y = np.zeros((nr, N), np.float64)
    lib().qgo_gemm_f64(_ptr(Xc), M, K, _ptr(Wc), N, _ptr(r), nr, _ptr(y))
    return y


# --------------------------------------------------------------------------
# INT8 outlier side path ("LLM inference cost: W8A8/W4A8 ...", sec. 2.2, second
# technique): the top 2% |w| of each group kept in INT8 beside the INT4 tile
# --------------------------------------------------------------------------
def outlier_count(group=128):
    """Outliers per group: ceil(2% of the group size) (3 of 128)."""
    return lib().qgo_outlier_count(int(group))


def outlier_split(W, group=128, count=None, s_smooth=None):
    """-> (idx u8 [G][count][N], codes8 i8 [G][count][N], s8 f32 [G][N], W_dense f32 [K][N], status)."""
    Wc = _c(W, np.float32)
    K, N = Wc.shape
    count = outlier_count(group) if count is None else int(count)
    G = K // group
    idx = np.zeros((G, count, N), np.uint8)
    c8 = np.zeros((G, count, N), np.int8)
    s8 = np.zeros((G, N), np.float32)
    dense = np.zeros((K, N), np.float32)
    ss = None if s_smooth is None else _c(s_smooth, np.float32)
    st = lib().qgo_outlier_split(_ptr(Wc), _ptr(ss), K, N, group, count, _ptr(idx), _ptr(c8), _ptr(s8), _ptr(dense))
    return idx, c8, s8, dense, st


def gemm_w4a16_outlier_ref(X, packed, scales, zeros, idx, codes8, s8, group=128, rows=None):
    """fp64 y = X deq4 + X deq8(outliers) and its |X||W| bound for the selected rows."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    p = _c(packed, np.uint32)
    N = p.shape[1]
    count = idx.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    y = np.zeros((nr, N), np.float64)
    b = np.zeros((nr, N), np.float64)
    lib().qgo_gemm_w4a16_outlier_ref(_ptr(Xc), M, K, N, _ptr(p), _ptr(_c(scales, np.uint16)), _ptr(_c(zeros, np.uint8)),
                                     group, count, _ptr(_c(idx, np.uint8)), _ptr(_c(codes8, np.int8)),
                                     _ptr(_c(s8, np.float32)), _ptr(r), nr, _ptr(y), _ptr(b))
    return y, b


# --------------------------------------------------------------------------
# 2:4 structured sparsity + INT4 ("LLM inference cost: W8A8/W4A8 ...", sec. 3.2):
# the 2 largest |w| of every 4 along K kept, then INT4 groups of 128
# --------------------------------------------------------------------------
def prune24(W):
    """-> (Wp f32 [K][N] with 2 of every 4 along K zeroed, meta u32 [K/32][N])."""
    Wc = _c(W, np.float32)
    K, N = Wc.shape
    Wp = np.zeros_like(Wc)
    meta = np.zeros((K // 32, N), np.uint32)
    lib().qgo_prune24(_ptr(Wc), K, N, _ptr(Wp), _ptr(meta))
    return Wp, meta


def pack24_vals(codes, meta):
    """Kept codes in k order, 8 per uint32 along K -> u32 [K/16][N]."""
    c = _c(codes, np.uint8)
    K, N = c.shape
    vals = np.zeros((K // 16, N), np.uint32)
    lib().qgo_pack24_vals(_ptr(c), _ptr(_c(meta, np.uint32)), K, N, _ptr(vals))
    return vals


def gemm_w4a16_24_ref(X, vals, meta, scales, zeros, group=128, rows=None):
    """fp64 y = X deq(2:4 sparse INT4 W) and its |X||W| bound for the selected rows."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    v = _c(vals, np.uint32)
    N = v.shape[1]
    r, nr = _rows(rows)
    nr = M if r is None else nr
    y = np.zeros((nr, N), np.float64)
    b = np.zeros((nr, N), np.float64)
    lib().qgo_gemm_w4a16_24_ref(_ptr(Xc), M, K, N, _ptr(v), _ptr(_c(meta, np.uint32)), _ptr(_c(scales, np.uint16)),
                                _ptr(_c(zeros, np.uint8)), group, _ptr(r), nr, _ptr(y), _ptr(b))
    return y, b


# --------------------------------------------------------------------------
# GPTQ ("Quantization & Flash Attention -- LLM inference optimization (2)", sec. 3.1-3.3):
# rows rounded one after another, each error spread over the later rows through the
# inverse Hessian (sequential OBS steps), stored in the asymmetric INT4 group format
# --------------------------------------------------------------------------
def gptq_hessian(X, damp=0.01):
    """H = (2/n) X^T X + lambda I, lambda = damp * mean diag -> f64 [K][K]."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    H = np.zeros((K, K), np.float64)
    lib().qgo_gptq_hessian(_ptr(Xc), M, K, float(damp), _ptr(H))
    return H


def gptq(X, W, group=128, damp=0.01):
    """-> (codes u8 [K][N], scales fp16 bits [K/g][N], zeros u8 [K/g][N], status)."""
    Xc = _c(X, np.float32)
    Wc = _c(W, np.float32)
    M, K = Xc.shape
    N = Wc.shape[1]
    codes = np.zeros((K, N), np.uint8)
    scales = np.zeros((K // group, N), np.uint16)
    zeros = np.zeros((K // group, N), np.uint8)
    st = lib().qgo_gptq(_ptr(Xc), M, K, _ptr(Wc), N, group, float(damp), _ptr(codes), _ptr(scales), _ptr(zeros))
    return codes, scales, zeros, st


def gptq_replay(X, W, codes, scales, zeros, group=128, damp=0.01, scale_ulps=1):
    """Teacher-forced replay of a given GPTQ result -> (code_slack, scale_miss, zero_miss, status)."""
    Xc = _c(X, np.float32)
    Wc = _c(W, np.float32)
    M, K = Xc.shape
    N = Wc.shape[1]
    slack = np.zeros(1, np.float64)
    sm = np.zeros(1, np.int64)
    zm = np.zeros(1, np.int64)
    st = lib().qgo_gptq_replay(_ptr(Xc), M, K, _ptr(Wc), N, group, float(damp), _ptr(_c(codes, np.uint8)),
                               _ptr(_c(scales, np.uint16)), _ptr(_c(zeros, np.uint8)), int(scale_ulps), _ptr(slack),
                               _ptr(sm), _ptr(zm))
    return float(slack[0]), int(sm[0]), int(zm[0]), st


# --------------------------------------------------------------------------
# AWQ scale search ("Quantization & Flash Attention -- LLM inference optimization (2)",
# sec. 2.1-2.3): s_c = mean|X_c|^alpha, alpha on a grid in [0, 1], least output MSE
# --------------------------------------------------------------------------
def awq_act_mean(X):
    """xm[c] = mean over tokens of |X[m][c]| (binary64 sum in token order, one rounding) -> f32 [K]."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    xm = np.zeros(K, np.float32)
    lib().qgo_awq_act_mean(_ptr(Xc), M, K, _ptr(xm))
    return xm


def awq_alpha(i, n_grid):
    """Grid point i of n_grid equally spaced points on [0, 1], both ends included."""
    return lib().qgo_awq_alpha(int(i), int(n_grid))


def awq_scales(xm, alpha):
    """s = xm^alpha (binary64 pow, one rounding; xm == 0 -> 1) and inv_s = 1/s -> (s, inv_s) f32 [K]."""
    x = _c(xm, np.float32)
    s = np.zeros_like(x)
    inv = np.zeros_like(x)
    lib().qgo_awq_scales(_ptr(x), x.size, float(alpha), _ptr(s), _ptr(inv))
    return s, inv


def awq_scale_act(X, inv_s):
    """X~ = bf16_rn(X * inv_s) -> bf16 bit patterns u16 [M][K]."""
    Xc = _c(X, np.float32)
    M, K = Xc.shape
    out = np.zeros((M, K), np.uint16)
    lib().qgo_awq_scale_act(_ptr(Xc), M, K, _ptr(_c(inv_s, np.float32)), _ptr(out))
    return out


def awq_candidate_mse(X, W, s, inv_s, group=128, yref=None):
    """MSE over all outputs of X W - bf16(X inv_s) deq(Q(diag(s) W)) -> (mse, status)."""
    Xc = _c(X, np.float32)
    Wc = _c(W, np.float32)
    M, K = Xc.shape
    N = Wc.shape[1]
    if yref is None:
        yref = gemm_f64(Xc, Wc)
    yref = _c(yref, np.float64)
    out = np.zeros(1, np.float64)
    st = lib().qgo_awq_candidate_mse(_ptr(Xc), M, K, _ptr(Wc), N, group, _ptr(_c(s, np.float32)),
                                     _ptr(_c(inv_s, np.float32)), _ptr(yref), _ptr(out))
    return float(out[0]), st


def awq_search(X, W, n_grid=21, group=128):
    """Grid search of alpha -> (mse f64 [n_grid], best index, s_best f32 [K], inv_s_best f32 [K], status)."""
    Xc = _c(X, np.float32)
    Wc = _c(W, np.float32)
    M, K = Xc.shape
    N = Wc.shape[1]
    mse = np.zeros(n_grid, np.float64)
    best = np.zeros(1, np.int32)
    s = np.zeros(K, np.float32)
    inv = np.zeros(K, np.float32)
    st = lib().qgo_awq_search(_ptr(Xc), M, K, _ptr(Wc), N, group, n_grid, _ptr(mse), _ptr(best), _ptr(s), _ptr(inv))
    return mse, int(best[0]), s, inv, st


def within_tolerance(y, yref, bound, rel=1e-2, abs_=1e-3):
    """The stated float bar: |y - y_ref| <= 1e-2 * (|X| |W_deq|) + 1e-3, elementwise."""
    return np.abs(np.asarray(y, np.float64) - yref) <= rel * bound + abs_


def build_variant(src_text: str, path: str):
    """Compile an edited copy of the oracle source to `path` and return its library handle.
    Used only by the tests that plant a mistake in the oracle to show the pins catch it."""
    src = path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-std=c11", "-fPIC",
                    "-shared", "-o", path, src, "-lm"], check=True)
    L = ctypes.CDLL(path)
    _declare(L)
    return L


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


class use_library:
    """Context manager: route this module's wrappers through another build of the oracle."""

    def __init__(self, L):
        self.L = L

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = self.L
        return self.L

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False
