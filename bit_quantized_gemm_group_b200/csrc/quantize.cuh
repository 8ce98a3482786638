// quantize.cuh -- offline weight quantizers, nibble packing, SmoothQuant factors.
//
// All of these are single HBM passes (they run once per weight load).  Every
// integer and every stored scale is produced in binary32 with round-to-nearest-even
// (__fdiv_rn / __fmul_rn / __float2int_rn), so the results are bit-identical to a
// plain IEEE implementation of the same formulas.
#pragma once
#include "common.cuh"

namespace qg {

// W~[k][n] = W[k][n] * s[k], one fp32 rounding (SmoothQuant, "AI Infra guide,
// ch.4 Quantization" sec. 2.2), or W itself.
QG_DEV_INLINE float smoothed_weight(const float* __restrict__ W, const float* __restrict__ s, int64_t N, int64_t k,
                                    int64_t n)
{
    float w = __ldg(W + k * N + n);
    return s ? __fmul_rn(w, __ldg(s + k)) : w;
}

// ---------------------------------------------------------------------------
// Group-wise asymmetric INT4 ("AI Infra guide, ch.4" sec. 1.1 affine quantization,
// sec. 1.2 asymmetric scale; group of 128 along K: "LLM inference cost" sec. 2.2).
// One thread per (group, column); a warp reads 32 adjacent columns of a row, so
// every row access is one coalesced 128-byte line.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_w4_asym_kernel(const float* __restrict__ W,
                                                                const float* __restrict__ s_smooth, int K, int N,
                                                                int group, uint8_t* __restrict__ codes,
                                                                uint16_t* __restrict__ scales,
                                                                uint8_t* __restrict__ zeros)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int64_t k0 = (int64_t)g * group;
    float mn = 0.0f, mx = 0.0f;  // the range always contains 0
    bool bad = false;
    for (int i = 0; i < group; ++i) {
        float v = smoothed_weight(W, s_smooth, N, k0 + i, n);
        bad |= !isfinite(v);
        if (v < mn) mn = v;
        if (v > mx) mx = v;
    }
    if (bad) { set_status(5u); return; }
    const float r = __fsub_rn(mx, mn);
    const float s32 = __fdiv_rn(r, 15.0f);
    if (s32 > 65504.0f) { set_status(6u); return; }
    __half s16 = __float2half_ru(s32);
    float s = __half2float(s16);
    int z = 0;
    if (r == 0.0f) {
        s16 = __ushort_as_half((unsigned short)0);
        s = 0.0f;
    } else {
        z = __float2int_rn(__fdiv_rn(-mn, s));
        z = min(max(z, 0), 15);
    }
    scales[(int64_t)g * N + n] = __half_as_ushort(s16);
    zeros[(int64_t)g * N + n] = (uint8_t)z;
    for (int i = 0; i < group; ++i) {
        int q = 0;
        if (s != 0.0f) {
            float v = smoothed_weight(W, s_smooth, N, k0 + i, n);
            q = __float2int_rn(__fdiv_rn(v, s)) + z;  // round(x/s) + z, in that order
            q = min(max(q, 0), 15);
        }
        codes[(k0 + i) * N + n] = (uint8_t)q;
    }
}

// ---------------------------------------------------------------------------
// Group-wise INT4, one HBM pass, for group in {64, 128, 256}: a CTA covers 128
// columns of one group; the group's rows are split in 4 quarters, one thread per
// (column, quarter) holding its GROUP/4 values in registers (a warp reads 128
// contiguous bytes of a row).  The quarters' range (or absmax) meet in shared memory;
// every thread of a column then derives the same scale and zero point with the same
// binary32 operations as the per-column kernels above, and quantizes from registers.
// ---------------------------------------------------------------------------
template <int GROUP, bool SYM>
__global__ void __launch_bounds__(512) quantize_w4_regs_kernel(const float* __restrict__ W,
                                                               const float* __restrict__ s_smooth, int K, int N,
                                                               uint8_t* __restrict__ codes, void* __restrict__ scales,
                                                               uint8_t* __restrict__ zeros)
{
    constexpr int RPT = GROUP / 4;  // rows per thread
    __shared__ float qmn[4][128], qmx[4][128];
    __shared__ int qbad[4][128];
    const int cl = threadIdx.x & 127, qr = threadIdx.x >> 7;
    const int n = blockIdx.x * 128 + cl;
    const int g = blockIdx.y;
    const int64_t k0 = (int64_t)g * GROUP + qr * RPT;
    const bool col_ok = n < N;
    float v[RPT];
    float mn = 0.0f, mx = 0.0f;  // asymmetric: the range always contains 0; symmetric: mx = max|w|
    bool bad = false;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        v[i] = col_ok ? smoothed_weight(W, s_smooth, N, k0 + i, n) : 0.0f;
        bad |= !isfinite(v[i]);
        if (SYM) {
            const float a = fabsf(v[i]);
            if (a > mx) mx = a;
        } else {
            if (v[i] < mn) mn = v[i];
            if (v[i] > mx) mx = v[i];
        }
    }
    qmn[qr][cl] = mn;
    qmx[qr][cl] = mx;
    qbad[qr][cl] = bad;
    __syncthreads();
    bool gbad = false;
    mn = 0.0f;
    mx = 0.0f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        gbad |= qbad[r][cl] != 0;
        if (qmn[r][cl] < mn) mn = qmn[r][cl];
        if (qmx[r][cl] > mx) mx = qmx[r][cl];
    }
    if (!col_ok) return;
    if (gbad) {
        if (qr == 0) set_status(5u);
        return;
    }
    uint8_t* crow = codes + k0 * N + n;
    if (SYM) {
        const float s = __fdiv_rn(mx, 7.0f);
        if (qr == 0) static_cast<float*>(scales)[(int64_t)g * N + n] = s;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            int q = 0;
            if (s != 0.0f) q = min(max(__float2int_rn(__fdiv_rn(v[i], s)), -7), 7);
            crow[(int64_t)i * N] = (uint8_t)(int8_t)q;
        }
    } else {
        const float r = __fsub_rn(mx, mn);
        const float s32 = __fdiv_rn(r, 15.0f);
        if (s32 > 65504.0f) {
            if (qr == 0) set_status(6u);
            return;
        }
        __half s16 = __float2half_ru(s32);
        float s = __half2float(s16);
        int z = 0;
        if (r == 0.0f) {
            s16 = __ushort_as_half((unsigned short)0);
            s = 0.0f;
        } else {
            z = min(max(__float2int_rn(__fdiv_rn(-mn, s)), 0), 15);
        }
        if (qr == 0) {
            static_cast<uint16_t*>(scales)[(int64_t)g * N + n] = __half_as_ushort(s16);
            zeros[(int64_t)g * N + n] = (uint8_t)z;
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            int q = 0;
            if (s != 0.0f) q = min(max(__float2int_rn(__fdiv_rn(v[i], s)) + z, 0), 15);  // round(x/s) + z
            crow[(int64_t)i * N] = (uint8_t)q;
        }
    }
}

// ---------------------------------------------------------------------------
// The same, with 16-byte accesses (N % 4 == 0): a CTA covers 128 columns of one group
// with 512 threads; thread (q, r) takes columns 4q .. 4q + 3 and rows r, r + 16, ..
// of the group, so a warp reads and writes whole 512-byte / 128-byte row segments.
// The 16 row slices' ranges meet in shared memory; one thread per column derives the
// scale and zero point (the binary32 operations of the per-column kernels) and every
// thread quantizes its values from registers.
// ---------------------------------------------------------------------------
template <int GROUP, bool SYM>
__global__ void __launch_bounds__(512, GROUP <= 128 ? 2 : 1) quantize_w4_vec_kernel(const float* __restrict__ W,
                                                              const float* __restrict__ s_smooth, int K, int N,
                                                              uint8_t* __restrict__ codes, void* __restrict__ scales,
                                                              uint8_t* __restrict__ zeros)
{
    constexpr int RPT = GROUP / 16;  // rows per thread
    __shared__ float qmn[16][128], qmx[16][128];
    __shared__ int qbad[16][128];
    __shared__ float fs[128];
    __shared__ int fz[128], fok[128];
    const int cq = threadIdx.x & 31, rr = threadIdx.x >> 5;
    const int n0 = blockIdx.x * 128 + 4 * cq;
    const int g = blockIdx.y;
    const bool quad_ok = n0 < N;  // N % 4 == 0: a quad is wholly inside or outside
    float v[RPT][4];
    float mn[4] = {0.f, 0.f, 0.f, 0.f}, mx[4] = {0.f, 0.f, 0.f, 0.f};  // asym: the range holds 0
    bool bad[4] = {false, false, false, false};
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int64_t k = (int64_t)g * GROUP + rr + 16 * i;
        float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
        if (quad_ok) w = __ldg(reinterpret_cast<const float4*>(W + k * N + n0));
        if (s_smooth) {
            const float sk = __ldg(s_smooth + k);
            w = make_float4(__fmul_rn(w.x, sk), __fmul_rn(w.y, sk), __fmul_rn(w.z, sk), __fmul_rn(w.w, sk));
        }
        v[i][0] = w.x; v[i][1] = w.y; v[i][2] = w.z; v[i][3] = w.w;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            bad[c] |= !isfinite(v[i][c]);
            if (SYM) {
                mx[c] = fmaxf(mx[c], fabsf(v[i][c]));
            } else {
                if (v[i][c] < mn[c]) mn[c] = v[i][c];
                if (v[i][c] > mx[c]) mx[c] = v[i][c];
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        qmn[rr][4 * cq + c] = mn[c];
        qmx[rr][4 * cq + c] = mx[c];
        qbad[rr][4 * cq + c] = bad[c];
    }
    __syncthreads();
    if (threadIdx.x < 128) {
        const int cl = threadIdx.x, n = blockIdx.x * 128 + cl;
        float a = 0.0f, b = 0.0f;
        bool gb = false;
        for (int r = 0; r < 16; ++r) {
            gb |= qbad[r][cl] != 0;
            if (qmn[r][cl] < a) a = qmn[r][cl];
            if (qmx[r][cl] > b) b = qmx[r][cl];
        }
        int ok = n < N && !gb;
        float sv = 0.0f;
        int zv = 0;
        if (n < N && gb) set_status(5u);
        if (ok) {
            if (SYM) {
                sv = __fdiv_rn(b, 7.0f);
                static_cast<float*>(scales)[(int64_t)g * N + n] = sv;
            } else {
                const float r = __fsub_rn(b, a);
                const float s32 = __fdiv_rn(r, 15.0f);
                if (s32 > 65504.0f) {
                    set_status(6u);
                    ok = 0;
                } else {
                    __half s16 = __float2half_ru(s32);
                    sv = __half2float(s16);
                    if (r == 0.0f) {
                        s16 = __ushort_as_half((unsigned short)0);
                        sv = 0.0f;
                    } else {
                        zv = min(max(__float2int_rn(__fdiv_rn(-a, sv)), 0), 15);
                    }
                    static_cast<uint16_t*>(scales)[(int64_t)g * N + n] = __half_as_ushort(s16);
                    zeros[(int64_t)g * N + n] = (uint8_t)zv;
                }
            }
        }
        fs[cl] = sv;
        fz[cl] = zv;
        fok[cl] = ok;
    }
    __syncthreads();
    if (!quad_ok) return;
    float sc[4];
    int zc[4], okc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        sc[c] = fs[4 * cq + c];
        zc[c] = fz[4 * cq + c];
        okc[c] = fok[4 * cq + c];
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int64_t k = (int64_t)g * GROUP + rr + 16 * i;
        uint32_t word = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            int q = 0;
            if (sc[c] != 0.0f) {
                if (SYM) q = min(max(__float2int_rn(__fdiv_rn(v[i][c], sc[c])), -7), 7);
                else q = min(max(__float2int_rn(__fdiv_rn(v[i][c], sc[c])) + zc[c], 0), 15);  // round(x/s) + z
            }
            word |= (uint32_t)(q & 0xFF) << (8 * c);
        }
        // a column whose group was not finite or overflowed keeps whatever its codes held
        uint8_t* dst = codes + k * N + n0;
        if (okc[0] && okc[1] && okc[2] && okc[3]) {
            *reinterpret_cast<uint32_t*>(dst) = word;
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (okc[c]) dst[c] = (uint8_t)(word >> (8 * c));
        }
    }
}

// Symmetric INT4: s = max|w|/7 (fp32), codes in [-7, 7] ("AI Infra guide, ch.4"
// sec. 1.2 symmetric scale, 4-bit analogue).
__global__ void __launch_bounds__(256) quantize_w4_sym_kernel(const float* __restrict__ W,
                                                               const float* __restrict__ s_smooth, int K, int N,
                                                               int group, int8_t* __restrict__ codes,
                                                               float* __restrict__ scales)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int64_t k0 = (int64_t)g * group;
    float amax = 0.0f;
    bool bad = false;
    for (int i = 0; i < group; ++i) {
        float v = smoothed_weight(W, s_smooth, N, k0 + i, n);
        bad |= !isfinite(v);
        float a = fabsf(v);
        if (a > amax) amax = a;
    }
    if (bad) { set_status(5u); return; }
    const float s = __fdiv_rn(amax, 7.0f);
    scales[(int64_t)g * N + n] = s;
    for (int i = 0; i < group; ++i) {
        int q = 0;
        if (s != 0.0f) {
            q = __float2int_rn(__fdiv_rn(smoothed_weight(W, s_smooth, N, k0 + i, n), s));
            q = min(max(q, -7), 7);
        }
        codes[(k0 + i) * N + n] = (int8_t)q;
    }
}

// ---------------------------------------------------------------------------
// Pack 8 codes per uint32 along K, low nibble first.  Each thread builds 4 words
// for 4 adjacent columns from 8 rows of 4-byte code loads and stores one uint4.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_nibbles_kernel(const uint8_t* __restrict__ codes, int K, int N,
                                                            uint32_t* __restrict__ packed)
{
    const int n4 = blockIdx.x * blockDim.x + threadIdx.x;  // group of 4 columns
    const int kb = blockIdx.y;
    if (n4 * 4 >= N) return;
    const int n = n4 * 4;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (n + 4 <= N && (N & 3) == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t c4 = __ldg(reinterpret_cast<const uint32_t*>(codes + (int64_t)(8 * kb + i) * N + n));
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] |= ((c4 >> (8 * j)) & 0xFu) << (4 * i);
        }
        *reinterpret_cast<uint4*>(packed + (int64_t)kb * N + n) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        for (int j = 0; j < 4 && n + j < N; ++j) {
            uint32_t wj = 0;
            for (int i = 0; i < 8; ++i) wj |= (uint32_t)(codes[(int64_t)(8 * kb + i) * N + n + j] & 0xF) << (4 * i);
            packed[(int64_t)kb * N + n + j] = wj;
        }
    }
}

// ---------------------------------------------------------------------------
// SmoothQuant factors ("AI Infra guide, ch.4" sec. 2.2).
// Pass 1a: ax[j] = max_m |Xcal[m][j]| (thread per column, coalesced rows) -> s[j]
// Pass 1b: aw[j] = max_n |W[j][n]| (block per row, tree reduction)       -> inv_s[j]
// Pass 2 : s[j] = ax^a / aw^(1-a), inv_s[j] = 1/s[j], in place.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) col_absmax_bf16_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                               float* __restrict__ out)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    float a = 0.0f;
    bool bad = false;
    for (int m = 0; m < M; ++m) {
        float v = bf16_bits_to_f32(__ldg(X + (int64_t)m * K + j));
        bad |= !isfinite(v);
        float av = fabsf(v);
        if (av > a) a = av;
    }
    if (bad) set_status(5u);
    out[j] = a;
}

__global__ void __launch_bounds__(256) row_absmax_f32_kernel(const float* __restrict__ W, int K, int N,
                                                              float* __restrict__ out)
{
    const int j = blockIdx.x;
    const float* row = W + (int64_t)j * N;
    float a = 0.0f;
    bool bad = false;
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        float v = __ldg(row + n);
        bad |= !isfinite(v);
        a = fmaxf(a, fabsf(v));
    }
    if (bad) set_status(5u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    __shared__ float red[32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x < 32) {
        a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (threadIdx.x == 0) out[j] = a;
    }
}

__global__ void smooth_finalize_kernel(float* __restrict__ s_io /*in: ax*/, float* __restrict__ inv_io /*in: aw*/,
                                       int K, float alpha)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const float ax = s_io[j], aw = inv_io[j];
    float sj;
    if (ax == 0.0f || aw == 0.0f)
        sj = 1.0f;
    else if (alpha == 0.5f)
        sj = __fdiv_rn(__fsqrt_rn(ax), __fsqrt_rn(aw));
    else
        sj = (float)(pow((double)ax, (double)alpha) / pow((double)aw, 1.0 - (double)alpha));
    s_io[j] = sj;
    inv_io[j] = __fdiv_rn(1.0f, sj);
}

// ---------------------------------------------------------------------------
// Per-output-channel symmetric INT8 ("AI Infra guide, ch.4" sec. 1.2-1.3) on
// W~ = diag(s) W: sw[n] = max_k |W~[k][n]| / 127, Wq = clamp(round(W~ / sw), -127, 127).
// ---------------------------------------------------------------------------
// Per-output-channel INT8 in two streaming passes (N % 4 == 0): pass 1 takes the column
// absmax of W~ = diag(s) W (|w| as integer bits, combined with atomicMax: the maximum of
// non-negative floats, exact in any order; non-finite values are reported and left
// out), pass 2 quantizes with sw = absmax / 127, and a last pass turns the absmax into
// sw in place.  Every pass is a CTA of 256 threads over 128 columns x 256 rows with
// 16-byte loads (a warp reads one 512-byte row segment) and 4-byte stores.  W is read
// twice: a one-read form (the rows of a column strip split over an 8-CTA cluster, held
// in shared memory, the absmax met through distributed shared memory) measured slower,
// held back by the cluster barrier per strip and by clusters of 8 filling 120 of 148 SMs,
// and so did running the passes over L2-sized column chunks.
__global__ void __launch_bounds__(256) w8_absmax_kernel(const float* __restrict__ W, const float* __restrict__ s,
                                                        int K, int N, unsigned int* __restrict__ amax_bits)
{
    __shared__ unsigned int part[8][128];
    const int cq = threadIdx.x & 31, rr = threadIdx.x >> 5;
    const int n0 = blockIdx.x * 128 + 4 * cq;
    const int k0 = blockIdx.y * 256;
    unsigned int a[4] = {0u, 0u, 0u, 0u};
    bool bad = false;
    if (n0 < N) {
#pragma unroll 8
        for (int i = 0; i < 32; ++i) {
            const int k = k0 + rr + 8 * i;
            if (k < K) {
                float4 w = __ldg(reinterpret_cast<const float4*>(W + (int64_t)k * N + n0));
                if (s) {
                    const float sk = __ldg(s + k);
                    w = make_float4(__fmul_rn(w.x, sk), __fmul_rn(w.y, sk), __fmul_rn(w.z, sk), __fmul_rn(w.w, sk));
                }
                const float v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (isfinite(v[c])) a[c] = max(a[c], __float_as_uint(fabsf(v[c])));
                    else bad = true;
                }
            }
        }
    }
    if (bad) set_status(5u);
#pragma unroll
    for (int c = 0; c < 4; ++c) part[rr][4 * cq + c] = a[c];
    __syncthreads();
    if (threadIdx.x < 128) {
        const int n = blockIdx.x * 128 + threadIdx.x;
        unsigned int m = 0u;
#pragma unroll
        for (int r = 0; r < 8; ++r) m = max(m, part[r][threadIdx.x]);
        if (n < N && m != 0u) atomicMax(amax_bits + n, m);
    }
}

__global__ void __launch_bounds__(256) w8_quant_kernel(const float* __restrict__ W, const float* __restrict__ s, int K,
                                                       int N, const unsigned int* __restrict__ amax_bits,
                                                       int8_t* __restrict__ Wq)
{
    const int cq = threadIdx.x & 31, rr = threadIdx.x >> 5;
    const int n0 = blockIdx.x * 128 + 4 * cq;
    const int k0 = blockIdx.y * 256;
    if (n0 >= N) return;
    const uint4 ab = *reinterpret_cast<const uint4*>(amax_bits + n0);
    const float sc[4] = {__fdiv_rn(__uint_as_float(ab.x), 127.0f), __fdiv_rn(__uint_as_float(ab.y), 127.0f),
                         __fdiv_rn(__uint_as_float(ab.z), 127.0f), __fdiv_rn(__uint_as_float(ab.w), 127.0f)};
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
        const int k = k0 + rr + 8 * i;
        if (k < K) {
            float4 w = __ldg(reinterpret_cast<const float4*>(W + (int64_t)k * N + n0));
            if (s) {
                const float sk = __ldg(s + k);
                w = make_float4(__fmul_rn(w.x, sk), __fmul_rn(w.y, sk), __fmul_rn(w.z, sk), __fmul_rn(w.w, sk));
            }
            const float v[4] = {w.x, w.y, w.z, w.w};
            uint32_t word = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                int q = 0;
                if (sc[c] != 0.0f && isfinite(v[c])) q = min(max(__float2int_rn(__fdiv_rn(v[c], sc[c])), -127), 127);
                word |= (uint32_t)(q & 0xFF) << (8 * c);
            }
            *reinterpret_cast<uint32_t*>(Wq + (int64_t)k * N + n0) = word;
        }
    }
}

__global__ void __launch_bounds__(256) w8_scale_kernel(float* __restrict__ sw, int N)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n < N) sw[n] = __fdiv_rn(__uint_as_float(__float_as_uint(sw[n])), 127.0f);
}

// ---------------------------------------------------------------------------
// Per-output-channel symmetric INT8, general shapes (any N, any K): one thread per
// column, pass 1 absmax, pass 2 quantize.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) quantize_w8_channel_kernel(const float* __restrict__ W,
                                                                   const float* __restrict__ s, int K, int N,
                                                                   int8_t* __restrict__ Wq, float* __restrict__ sw)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float a = 0.0f;
    bool bad = false;
    for (int k = 0; k < K; ++k) {
        float v = smoothed_weight(W, s, N, k, n);
        bad |= !isfinite(v);
        float av = fabsf(v);
        if (av > a) a = av;
    }
    if (bad) set_status(5u);
    const float sc = __fdiv_rn(a, 127.0f);
    sw[n] = sc;
    for (int k = 0; k < K; ++k) {
        int q = 0;
        float v = smoothed_weight(W, s, N, k, n);
        if (sc != 0.0f && isfinite(v)) q = min(max(__float2int_rn(__fdiv_rn(v, sc)), -127), 127);
        Wq[(int64_t)k * N + n] = (int8_t)q;
    }
}

}  // namespace qg
