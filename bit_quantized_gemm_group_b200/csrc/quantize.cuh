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
// W~ = diag(s) W, one HBM pass: a strip of 8 columns (32-byte row segments) is
// split along K over the CTAs of a thread-block cluster (up to 8), each CTA holding
// its rows of the strip in registers (4 rows x 8 columns per thread, 2048 rows per
// CTA).  The column absmax (exact in any order) is reduced within the CTA with warp
// shuffles, then across the cluster through distributed shared memory; each CTA then
// quantizes the values it holds.  For N % 8 == 0 and K <= 16384.
// ---------------------------------------------------------------------------
constexpr int kW8StripThreads = 512;
constexpr int kW8StripRowsPerThread = 4;
constexpr int kW8StripRows = kW8StripThreads * kW8StripRowsPerThread;  // rows of K per CTA

__global__ void __launch_bounds__(kW8StripThreads) quantize_w8_strip_kernel(const float* __restrict__ W,
                                                                            const float* __restrict__ s, int K,
                                                                            int N, int8_t* __restrict__ Wq,
                                                                            float* __restrict__ sw)
{
    __shared__ float wmax[kW8StripThreads / 32][8];
    __shared__ __align__(16) float cmax[8];
    const int n0 = 8 * blockIdx.x;
    const uint32_t rank = cluster_ctarank();
    const int C = (int)gridDim.y;  // the whole y extent is one cluster
    const int kb = (int)((int64_t)K * rank / C), ke = (int)((int64_t)K * (rank + 1) / C);
    float v[kW8StripRowsPerThread][8];
    float a[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) a[c] = 0.0f;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < kW8StripRowsPerThread; ++i) {
        const int k = kb + (int)threadIdx.x + kW8StripThreads * i;
        if (k < ke) {
            const float4* src = reinterpret_cast<const float4*>(W + (int64_t)k * N + n0);
            const float4 lo = __ldg(src), hi = __ldg(src + 1);
            const float sk = s ? __ldg(s + k) : 1.0f;
            const float raw[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                v[i][c] = s ? __fmul_rn(raw[c], sk) : raw[c];
                bad |= !isfinite(v[i][c]);
                a[c] = fmaxf(a[c], fabsf(v[i][c]));
            }
        } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) v[i][c] = 0.0f;
        }
    }
    if (bad) set_status(5u);
    // CTA absmax per column
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a[c] = fmaxf(a[c], __shfl_xor_sync(0xffffffffu, a[c], o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
#pragma unroll
        for (int c = 0; c < 8; ++c) wmax[warp][c] = a[c];
    __syncthreads();
    if (threadIdx.x < 8) {
        float m = 0.0f;
        for (int w = 0; w < kW8StripThreads / 32; ++w) m = fmaxf(m, wmax[w][threadIdx.x]);
        cmax[threadIdx.x] = m;
    }
    // cluster absmax per column through distributed shared memory
    cluster_sync();
    if (threadIdx.x < 8) {
        float m = 0.0f;
        const uint32_t la = smem_u32(&cmax[threadIdx.x]);
        for (int r = 0; r < C; ++r) m = fmaxf(m, ld_dsmem_f32(dsmem_addr(la, (uint32_t)r)));
        wmax[0][threadIdx.x] = __fdiv_rn(m, 127.0f);  // the column scale
    }
    cluster_sync();  // every CTA has read every cmax before any CTA moves on
    float sc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) sc[c] = wmax[0][c];
    if (rank == 0 && threadIdx.x < 8 && n0 + (int)threadIdx.x < N) sw[n0 + threadIdx.x] = sc[threadIdx.x];
#pragma unroll
    for (int i = 0; i < kW8StripRowsPerThread; ++i) {
        const int k = kb + (int)threadIdx.x + kW8StripThreads * i;
        if (k < ke) {
            uint32_t lo = 0, hi = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                int q = 0;
                if (sc[c] != 0.0f && isfinite(v[i][c])) q = min(max(__float2int_rn(__fdiv_rn(v[i][c], sc[c])), -127), 127);
                const uint32_t b = (uint32_t)(q & 0xFF) << (8 * (c & 3));
                if (c < 4) lo |= b;
                else hi |= b;
            }
            *reinterpret_cast<uint2*>(Wq + (int64_t)k * N + n0) = make_uint2(lo, hi);
        }
    }
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
