// act_quant.cuh -- fused smoothing + per-token absmax + INT8 quantization.
//
// "AI Infra guide, ch.4 Quantization": sec. 2.2 (X~ = X diag(s)^-1), sec. 1.2
// (symmetric s = max|x|/127), sec. 1.3 (per-token dynamic scale).
//
// One CTA per token row.  Pass 1 streams the row from HBM with 16-byte loads
// (8 bf16 per thread per chunk), multiplies by inv_s and reduces |X~| with warp
// shuffles and one shared-memory step; pass 2 re-reads the row (an L1 hit: a row
// is at most a few tens of KB) and writes 8 int8 codes per thread per chunk.
// Bytes from HBM per element: 2 read + 1 written.
#pragma once
#include "common.cuh"

namespace qg {

QG_DEV_INLINE void load_smoothed8(const uint16_t* __restrict__ xrow, const float* __restrict__ inv_s, int j,
                                  float (&v)[8])
{
    const uint4 raw = ldg_v4(xrow + j);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    if (inv_s) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(inv_s + j));
        const float4 b = __ldg(reinterpret_cast<const float4*>(inv_s + j + 4));
        v[0] = __fmul_rn(v[0], a.x);
        v[1] = __fmul_rn(v[1], a.y);
        v[2] = __fmul_rn(v[2], a.z);
        v[3] = __fmul_rn(v[3], a.w);
        v[4] = __fmul_rn(v[4], b.x);
        v[5] = __fmul_rn(v[5], b.y);
        v[6] = __fmul_rn(v[6], b.z);
        v[7] = __fmul_rn(v[7], b.w);
    }
}

__global__ void __launch_bounds__(256) smooth_quant_act_i8_kernel(const uint16_t* __restrict__ X, int K,
                                                                   const float* __restrict__ inv_s,
                                                                   int8_t* __restrict__ Xq, float* __restrict__ t)
{
    const int64_t m = blockIdx.x;
    const uint16_t* xrow = X + m * K;
    float a = 0.0f;
    bool bad = false;
    for (int j = threadIdx.x * 8; j < K; j += blockDim.x * 8) {
        float v[8];
        load_smoothed8(xrow, inv_s, j, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            bad |= !isfinite(v[i]);
            a = fmaxf(a, fabsf(v[i]));
        }
    }
    if (bad) set_status(5u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    __shared__ float red[32];
    __shared__ float t_sh;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x < 32) {
        a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (threadIdx.x == 0) {
            const float tm = __fdiv_rn(a, 127.0f);
            t_sh = tm;
            t[m] = tm;
        }
    }
    __syncthreads();
    const float tm = t_sh;
    int8_t* qrow = Xq + m * K;
    for (int j = threadIdx.x * 8; j < K; j += blockDim.x * 8) {
        float v[8];
        load_smoothed8(xrow, inv_s, j, v);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int q = 0;
            if (tm != 0.0f && isfinite(v[i])) q = min(max(__float2int_rn(__fdiv_rn(v[i], tm)), -127), 127);
            const uint32_t b = (uint32_t)(q & 0xFF);
            if (i < 4) lo |= b << (8 * i);
            else hi |= b << (8 * (i - 4));
        }
        *reinterpret_cast<uint2*>(qrow + j) = make_uint2(lo, hi);
    }
}

}  // namespace qg
