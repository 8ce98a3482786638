// awq.cuh -- activation-aware scales for the INT4 weights (AWQ): the per-channel
// statistic, the scales for one grid point, the scaled activations, the layer's
// reference output and the output error of one candidate.
//
// "Quantization & Flash Attention -- LLM inference optimization (2)":
//   sec. 2.1  statistic: mean magnitude E[|X_c|] of each input channel over a
//             calibration batch;
//   sec. 2.2  equivalent transform X W = (X / s)(s W), one s per input channel;
//   sec. 2.3  s_c = mean(|X_c|)^alpha, alpha on a grid in [0, 1], the one whose
//             quantized layer output is closest (MSE) to X W.
// The search itself (one pass of quantize -> pack -> W4A16 GEMM -> error per grid
// point, all on the stream) is driven by qg_awq_search in qgemm.cu; these kernels are
// the steps the INT4 path does not already have.  Every step is a single pass over
// HBM or a small reduction; the GEMMs are the heavy part.
#pragma once
#include "common.cuh"

namespace qg {

// xm[c] = (float)((sum over m, in order, of |X[m][c]| in binary64) / M).  One thread
// per channel walks the tokens in order, so the binary64 sum, and hence xm, is the
// same on every run and for every launch shape.  A warp reads 32 adjacent channels
// of one token (64 contiguous bytes) per step.
__global__ void __launch_bounds__(256) awq_act_mean_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                           float* __restrict__ xm)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= K) return;
    double sum = 0.0;
    for (int m = 0; m < M; ++m) sum += fabs((double)bf16_bits_to_f32(__ldg(X + (int64_t)m * K + c)));
    xm[c] = (float)(sum / (double)M);
}

// s[c] = (float)pow((double)xm[c], alpha) and a zero statistic keeps s[c] = 1;
// inv_s[c] = 1 / s[c] in binary32, round to nearest.  With `idx_dev` given, alpha is
// the grid point alpha_i = i / (n_grid - 1) (both ends included; 0 when n_grid == 1)
// of the index stored there (the search's winner); otherwise `alpha` itself.
__global__ void __launch_bounds__(256) awq_scales_kernel(const float* __restrict__ xm, int K, double alpha_given,
                                                         const int32_t* __restrict__ idx_dev, int n_grid,
                                                         float* __restrict__ s, float* __restrict__ inv_s)
{
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= K) return;
    const double alpha = !idx_dev ? alpha_given : n_grid > 1 ? (double)*idx_dev / (double)(n_grid - 1) : 0.0;
    const float x = xm[c];
    const float sc = x == 0.0f ? 1.0f : (float)pow((double)x, alpha);
    s[c] = sc;
    inv_s[c] = __fdiv_rn(1.0f, sc);
}

// Xs[m][k] = bf16_rn(X[m][k] * inv_s[k]) (binary32 product, rounded once to bf16):
// the scaled activations in the layer's activation dtype.  Eight elements (16 bytes)
// per thread step, grid-stride.  Requires K % 8 == 0.
__global__ void __launch_bounds__(256) awq_scale_act_kernel(const uint16_t* __restrict__ X, int64_t total8, int K,
                                                            const float* __restrict__ inv_s, uint16_t* __restrict__ Xs)
{
    for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total8; v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e0 = v * 8;
        const int k0 = (int)(e0 % K);
        const uint4 in = __ldg(reinterpret_cast<const uint4*>(X + e0));
        const float4 i0 = __ldg(reinterpret_cast<const float4*>(inv_s + k0));
        const float4 i1 = __ldg(reinterpret_cast<const float4*>(inv_s + k0 + 4));
        const uint32_t w[4] = {in.x, in.y, in.z, in.w};
        const float f[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __fmul_rn(bf16_bits_to_f32(w[j] & 0xFFFFu), f[2 * j]);
            const float hi = __fmul_rn(bf16_bits_to_f32(w[j] >> 16), f[2 * j + 1]);
            o[j] = (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
        }
        *reinterpret_cast<uint4*>(Xs + e0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Yref[m][n] = sum_k X[m][k] W[k][n]: bf16 activations times the unquantized fp32
// weights, fp32 fused multiply-adds in k order.  The reference output of the
// search: computed once per search, so a plain shared-memory tiled SIMT kernel
// (64 x 64 outputs per CTA, 4 x 4 per thread, k steps of 16) is enough next to the
// per-candidate work.  Requires K % 16 == 0.
constexpr int kAwqRefBM = 64, kAwqRefBN = 64, kAwqRefBK = 16;

__global__ void __launch_bounds__(256) awq_ref_gemm_kernel(const uint16_t* __restrict__ X, const float* __restrict__ W,
                                                           int M, int K, int N, float* __restrict__ Y)
{
    // As[k][m] (rows padded by 4 floats: the transposing stores spread over the banks),
    // Bs[k][n]; both read as float4 along m / n
    __shared__ __align__(16) float As[kAwqRefBK][kAwqRefBM + 4];
    __shared__ __align__(16) float Bs[kAwqRefBK][kAwqRefBN];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * kAwqRefBM, n0 = blockIdx.x * kAwqRefBN;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    for (int k0 = 0; k0 < K; k0 += kAwqRefBK) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int e = tid + 256 * r;
            const int am = e >> 4, ak = e & 15;  // 64 rows x 16 k
            As[ak][am] = m0 + am < M ? bf16_bits_to_f32(__ldg(X + (int64_t)(m0 + am) * K + k0 + ak)) : 0.0f;
            const int bk = e >> 6, bn = e & 63;  // 16 k x 64 columns
            Bs[bk][bn] = n0 + bn < N ? __ldg(W + (int64_t)(k0 + bk) * N + n0 + bn) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kAwqRefBK; ++kk) {
            const float4 av = *reinterpret_cast<const float4*>(&As[kk][4 * ty]);
            const float4 bv = *reinterpret_cast<const float4*>(&Bs[kk][4 * tx]);
            const float a[4] = {av.x, av.y, av.z, av.w}, b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + 4 * tx + j;
            if (n < N) Y[(int64_t)m * N + n] = acc[i][j];
        }
    }
}

// Sum of squared differences (Yref - Yq)^2 in binary64 over `count` outputs, Yq in
// bf16.  A fixed grid of kAwqErrBlocks CTAs; thread t of CTA b takes elements
// b*256 + t + j*(256 * kAwqErrBlocks), and each CTA reduces its threads in a fixed
// tree, so the partial sums (and the MSE built from them) do not vary between runs.
constexpr int kAwqErrBlocks = 256;

__global__ void __launch_bounds__(256) awq_sqerr_kernel(const float* __restrict__ Yref, const uint16_t* __restrict__ Yq,
                                                        int64_t count, double* __restrict__ partials)
{
    __shared__ double red[256];
    double acc = 0.0;
    for (int64_t i = blockIdx.x * 256 + threadIdx.x; i < count; i += 256 * (int64_t)kAwqErrBlocks) {
        const double d = (double)__ldg(Yref + i) - (double)bf16_bits_to_f32(__ldg(Yq + i));
        acc = fma(d, d, acc);
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) partials[blockIdx.x] = red[0];
}

// mse_i = (sum of the partials, in CTA order) / count.  One thread.
__global__ void awq_mse_finish_kernel(const double* __restrict__ partials, int64_t count, double* __restrict__ mse_i)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double s = 0.0;
    for (int b = 0; b < kAwqErrBlocks; ++b) s += partials[b];
    *mse_i = s / (double)count;
}

// best = the first grid index with the least MSE.  One thread.
__global__ void awq_argmin_kernel(const double* __restrict__ mse, int n_grid, int32_t* __restrict__ best)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int b = 0;
    for (int i = 1; i < n_grid; ++i)
        if (mse[i] < mse[b]) b = i;
    *best = b;
}

}  // namespace qg
