// gptq.cuh -- GPTQ: INT4 weights with Hessian-weighted error compensation.
//
// "Quantization & Flash Attention -- LLM inference optimization (2)", sec. 3.1-3.3: the
// rows of W (input channels) are rounded one after another; the error of each is spread
// over the rows not yet rounded through the inverse Hessian H^-1, H = (2/n) X^T X +
// lambda I over n calibration tokens (Optimal Brain Surgeon steps).
//
// The device path takes the same steps in the same order as their plain definition,
// with every binary64 / binary32 operation rounded on its own (the _rn intrinsics: no
// fused multiply-add contraction), so its codes, scales and zeros are those of the
// definition bit for bit:
//   H[a][b]  = (2 (sum over tokens, in order, of x_a x_b)) / n, then + lambda on the
//              diagonal, lambda = damp * trace / K (trace summed in order);
//   H^-1     by Gauss-Jordan without pivoting (H is symmetric positive definite):
//              per column c, row c divided by its pivot, then every other row r
//              minus a[r][c] times row c;
//   rows k   in order: at a group's first row, its scale and zero (the asymmetric INT4
//              rules) from the group's compensated weights rounded to binary32; the
//              row's codes; e = (w - deq) / Hinv[k][k]; w_j -= e Hinv[k][j] for j > k;
//              then row and column k eliminated from Hinv.
// Each step is one elementwise or row kernel; the work is O(K^3 + K^2 N) binary64
// operations, an offline cost (once per weight matrix).
#pragma once
#include "common.cuh"

namespace qg {

// H[a][b] = (2 * sum_m x[m][a] x[m][b]) / Mc; one thread per (a, b), tokens in order.
__global__ void __launch_bounds__(256) gptq_hessian_kernel(const uint16_t* __restrict__ X, int Mc, int K,
                                                           double* __restrict__ H)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    const int a = blockIdx.y;
    if (b >= K) return;
    double s = 0.0;
    for (int m = 0; m < Mc; ++m) {
        const double xa = (double)bf16_bits_to_f32(__ldg(X + (int64_t)m * K + a));
        const double xb = (double)bf16_bits_to_f32(__ldg(X + (int64_t)m * K + b));
        s = __dadd_rn(s, __dmul_rn(xa, xb));
    }
    H[(int64_t)a * K + b] = __ddiv_rn(__dmul_rn(2.0, s), (double)Mc);
}

// lambda = damp * trace / K (damp alone when the trace is 0), added to the diagonal.
// One thread: the trace is summed in index order.
__global__ void gptq_ridge_kernel(double* __restrict__ H, int K, double damp)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double tr = 0.0;
    for (int a = 0; a < K; ++a) tr = __dadd_rn(tr, H[(int64_t)a * K + a]);
    const double lambda = tr > 0.0 ? __ddiv_rn(__dmul_rn(damp, tr), (double)K) : damp;
    for (int a = 0; a < K; ++a) H[(int64_t)a * K + a] = __dadd_rn(H[(int64_t)a * K + a], lambda);
}

// inv = identity
__global__ void __launch_bounds__(256) gptq_identity_kernel(double* __restrict__ inv, int K)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int i = blockIdx.y;
    if (j < K) inv[(int64_t)i * K + j] = i == j ? 1.0 : 0.0;
}

// Gauss-Jordan step c, part 1: f[r] = a[r][c] for every row (f[c] is the pivot).
__global__ void __launch_bounds__(256) gj_column_kernel(const double* __restrict__ a, int K, int c,
                                                        double* __restrict__ f)
{
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r < K) f[r] = a[(int64_t)r * K + c];
}

// part 2: row c of a and of inv divided by the pivot f[c] (a zero pivot is recorded).
__global__ void __launch_bounds__(256) gj_scale_kernel(double* __restrict__ a, double* __restrict__ inv, int K, int c,
                                                       const double* __restrict__ f)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const double d = f[c];
    if (d == 0.0) {
        if (j == 0) set_status(6u);
        return;
    }
    a[(int64_t)c * K + j] = __ddiv_rn(a[(int64_t)c * K + j], d);
    inv[(int64_t)c * K + j] = __ddiv_rn(inv[(int64_t)c * K + j], d);
}

// part 3: every row r != c minus f[r] times row c (row c and f are only read).
__global__ void __launch_bounds__(256) gj_eliminate_kernel(double* __restrict__ a, double* __restrict__ inv, int K,
                                                           int c, const double* __restrict__ f)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int r = blockIdx.y;
    if (j >= K || r == c) return;
    const double fr = f[r];
    a[(int64_t)r * K + j] = __dsub_rn(a[(int64_t)r * K + j], __dmul_rn(fr, a[(int64_t)c * K + j]));
    inv[(int64_t)r * K + j] = __dsub_rn(inv[(int64_t)r * K + j], __dmul_rn(fr, inv[(int64_t)c * K + j]));
}

// Wc = (double)W; a non-finite weight is recorded.
__global__ void __launch_bounds__(256) gptq_load_kernel(const float* __restrict__ W, int64_t total,
                                                        double* __restrict__ Wc)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const float w = __ldg(W + i);
        if (!isfinite(w)) set_status(5u);
        Wc[i] = (double)w;
    }
}

// At a group's first row k: scale and zero of each column's group from the compensated
// weights rounded to binary32 (range widened to contain 0, s = fp16 rounded up of
// r / 15, z = round(-min / s) clamped to [0, 15]; a zero range gives 0 and 0).
__global__ void __launch_bounds__(256) gptq_group_kernel(const double* __restrict__ Wc, int N, int k, int group,
                                                         uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros,
                                                         float* __restrict__ s_col, int* __restrict__ z_col)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float mn = 0.0f, mx = 0.0f;
    for (int i = 0; i < group; ++i) {
        const float v = __double2float_rn(Wc[(int64_t)(k + i) * N + n]);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    const float r = __fsub_rn(mx, mn);
    const float s32 = __fdiv_rn(r, 15.0f);
    if (s32 > 65504.0f) set_status(6u);
    __half s16 = __float2half_ru(s32);
    float s = __half2float(s16);
    int z = 0;
    if (r == 0.0f) {
        s16 = __ushort_as_half((unsigned short)0);
        s = 0.0f;
    } else {
        z = min(max(__float2int_rn(__fdiv_rn(-mn, s)), 0), 15);
    }
    const int g = k / group;
    scales[(int64_t)g * N + n] = __half_as_ushort(s16);
    zeros[(int64_t)g * N + n] = (uint8_t)z;
    s_col[n] = s;
    z_col[n] = z;
}

// Row k: its codes, and e[n] = (w - (q - z) s) / Hinv[k][k].
__global__ void __launch_bounds__(256) gptq_row_kernel(const double* __restrict__ Wc, int K, int N, int k,
                                                       const double* __restrict__ Hinv,
                                                       const float* __restrict__ s_col, const int* __restrict__ z_col,
                                                       uint8_t* __restrict__ codes, double* __restrict__ e)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const double wd = Wc[(int64_t)k * N + n];
    const float w = __double2float_rn(wd);
    const float s = s_col[n];
    const int z = z_col[n];
    const int q = s != 0.0f ? min(max(__float2int_rn(__fdiv_rn(w, s)) + z, 0), 15) : 0;
    codes[(int64_t)k * N + n] = (uint8_t)q;
    e[n] = __ddiv_rn(__dsub_rn(wd, __dmul_rn((double)(q - z), (double)s)), Hinv[(int64_t)k * K + k]);
}

// Rows j > k: w_j -= e Hinv[k][j].
__global__ void __launch_bounds__(256) gptq_update_kernel(double* __restrict__ Wc, int K, int N, int k,
                                                          const double* __restrict__ Hinv, const double* __restrict__ e)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int j = k + 1 + blockIdx.y;
    if (n >= N || j >= K) return;
    Wc[(int64_t)j * N + n] = __dsub_rn(Wc[(int64_t)j * N + n], __dmul_rn(e[n], Hinv[(int64_t)k * K + j]));
}

// Eliminate row and column k: for a, b > k, Hinv[a][b] -= (Hinv[a][k] / Hinv[k][k]) Hinv[k][b]
// (column k and row k are only read).
__global__ void __launch_bounds__(256) gptq_eliminate_kernel(double* __restrict__ Hinv, int K, int k)
{
    const int b = k + 1 + blockIdx.x * blockDim.x + threadIdx.x;
    const int a = k + 1 + blockIdx.y;
    if (b >= K || a >= K) return;
    const double f = __ddiv_rn(Hinv[(int64_t)a * K + k], Hinv[(int64_t)k * K + k]);
    Hinv[(int64_t)a * K + b] = __dsub_rn(Hinv[(int64_t)a * K + b], __dmul_rn(f, Hinv[(int64_t)k * K + b]));
}

}  // namespace qg
