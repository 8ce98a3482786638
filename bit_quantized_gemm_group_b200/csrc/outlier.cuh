// outlier.cuh -- the INT8 outlier side path beside the INT4 groups.
//
// "LLM inference cost: W8A8/W4A8 ...", sec. 2.2, second technique: at calibration time
// the largest-magnitude 2% of each group's weights are found and kept in INT8 apart
// from the INT4 tile; at run time their product is computed on a side path and added
// to the INT4 product.
//   split:    per (group g, column n) the `count` weights of largest |w| (ties: smaller
//             k first), stored as k offset (u8) + symmetric INT8 code with one fp32
//             scale s8 = max|outlier| / 127; the remainder (outliers set to 0) goes to
//             the ordinary asymmetric INT4 quantizer.
//   side add: Y[m][n] += sum over the outliers of X[m][k] * code * s8.
// Layouts: idx u8 [G][count][N], codes8 i8 [G][count][N], s8 fp32 [G][N]; all
// coalesced along N, like the INT4 scales and zeros.
#pragma once
#include "common.cuh"
#include "quantize.cuh"

namespace qg {

constexpr int kMaxOutliers = 8;  // per group; 2% of a group of up to 400

// One thread per (group, column): a warp reads 32 adjacent columns of a row (one
// 128-byte line).  The running top-`count` list is kept sorted (|w| descending, then
// k ascending) by insertion: an element enters at the first slot it strictly exceeds
// and every later slot shifts down one.
__global__ void __launch_bounds__(256) outlier_split_kernel(const float* __restrict__ W,
                                                            const float* __restrict__ s_smooth, int K, int N,
                                                            int group, int count, uint8_t* __restrict__ idx,
                                                            int8_t* __restrict__ codes8, float* __restrict__ s8,
                                                            float* __restrict__ W_dense)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int g = blockIdx.y;
    if (n >= N) return;
    const int64_t k0 = (int64_t)g * group;
    float ta[kMaxOutliers], tv[kMaxOutliers];
    int ti[kMaxOutliers];
#pragma unroll
    for (int j = 0; j < kMaxOutliers; ++j) {
        ta[j] = -1.0f;
        tv[j] = 0.0f;
        ti[j] = 0;
    }
    bool bad = false;
    for (int i = 0; i < group; ++i) {
        float v = smoothed_weight(W, s_smooth, N, k0 + i, n);
        bad |= !isfinite(v);
        float a = fabsf(v);
        int k = i;
        bool shift = false;
#pragma unroll
        for (int j = 0; j < kMaxOutliers; ++j) {
            if (j < count && (shift || a > ta[j])) {
                const float ta0 = ta[j], tv0 = tv[j];
                const int ti0 = ti[j];
                ta[j] = a;
                tv[j] = v;
                ti[j] = k;
                a = ta0;
                v = tv0;
                k = ti0;
                shift = true;
            }
        }
    }
    if (bad) {
        set_status(5u);
        return;
    }
    const float sc = count > 0 ? __fdiv_rn(ta[0], 127.0f) : 0.0f;
    s8[(int64_t)g * N + n] = sc;
#pragma unroll
    for (int j = 0; j < kMaxOutliers; ++j) {
        if (j < count) {
            int q = 0;
            if (sc != 0.0f) q = min(max(__float2int_rn(__fdiv_rn(tv[j], sc)), -127), 127);
            idx[((int64_t)g * count + j) * N + n] = (uint8_t)ti[j];
            codes8[((int64_t)g * count + j) * N + n] = (int8_t)q;
        }
    }
    // the remainder: the group's values with the outliers set to 0
    for (int i = 0; i < group; ++i) {
        bool out = false;
#pragma unroll
        for (int j = 0; j < kMaxOutliers; ++j) out |= (j < count && ti[j] == i);
        W_dense[(k0 + i) * N + n] = out ? 0.0f : smoothed_weight(W, s_smooth, N, k0 + i, n);
    }
}

// Y[m][n] = rn(Y[m][n] + sum_{g, r} X[m][g*group + idx] * (code * s8[g][n])), in fp32 with
// one rounding back to the output dtype.  One thread per column and a chunk of MT
// tokens; idx, codes and scales are read once per chunk (coalesced along N); the
// gathered X elements come from L1/L2 (X is small next to the weights).
template <int MT, bool BF16>
__global__ void __launch_bounds__(128) outlier_side_add_kernel(const uint16_t* __restrict__ X, int M, int K, int N,
                                                               int group, int count, const uint8_t* __restrict__ idx,
                                                               const int8_t* __restrict__ codes8,
                                                               const float* __restrict__ s8, uint16_t* __restrict__ Y)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int m0 = blockIdx.y * MT;
    if (n >= N) return;
    const int G = K / group;
    float acc[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
    bool bad = false;
    for (int g = 0; g < G; ++g) {
        const float sc = __ldg(s8 + (int64_t)g * N + n);
        for (int r = 0; r < count; ++r) {
            const int64_t o = ((int64_t)g * count + r) * N + n;
            const int off = (int)__ldg(idx + o);
            if (off >= group) {  // not an offset inside the group: skipped and reported
                bad = true;
                continue;
            }
            const int k = g * group + off;
            const float w = __fmul_rn((float)__ldg(codes8 + o), sc);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (m0 + t < M) {
                    const uint16_t xb = __ldg(X + (int64_t)(m0 + t) * K + k);
                    const float x = BF16 ? bf16_bits_to_f32(xb) : __half2float(__ushort_as_half(xb));
                    acc[t] = fmaf(x, w, acc[t]);
                }
            }
        }
    }
    if (bad) set_status(6u);
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        if (m0 + t < M) {
            uint16_t* y = Y + (int64_t)(m0 + t) * N + n;
            if (BF16) {
                *y = f32_to_bf16_bits(__fadd_rn(bf16_bits_to_f32(*y), acc[t]));
            } else {
                *y = f32_to_f16_bits(__fadd_rn(__half2float(__ushort_as_half(*y)), acc[t]));
            }
        }
    }
}

}  // namespace qg
