// sparse24.cuh -- 2:4 structured sparsity + INT4 weights.
//
// "LLM inference cost: W8A8/W4A8 ...", sec. 3.2: in every 4 consecutive weights along K
// the 2 of largest |w| are kept (ties: smaller k), the other 2 become 0; the kept
// weights are quantized to asymmetric INT4 in groups of 128 (the ordinary quantizer on
// the pruned matrix).  Storage: the kept codes in k order, 8 per uint32 along K
// (vals [K/16][N], two per 4-block), and the kept positions i0 < i1 of 4-block b as
// the nibble (i1 << 2) | i0 at bits 4 (b mod 8) of meta[b / 8][n] ([K/32][N]): 0.375
// bytes per weight with the positions, against 0.5 for dense INT4.
#pragma once
#include "common.cuh"

namespace qg {

// One thread per (column, 8 blocks = 32 rows): one metadata word.  A warp reads 32
// adjacent columns of a row (one 128-byte line).
__global__ void __launch_bounds__(256) prune24_kernel(const float* __restrict__ W, int K, int N,
                                                      float* __restrict__ Wp, uint32_t* __restrict__ meta)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int kw = blockIdx.y;  // metadata word: rows 32 kw .. 32 kw + 31
    if (n >= N) return;
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const int64_t k0 = 32 * (int64_t)kw + 4 * b;
        float v[4], a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[i] = __ldg(W + (k0 + i) * N + n);
            a[i] = fabsf(v[i]);
        }
        // the largest |w| (first on ties), then the largest of the other three
        int p0 = 0;
#pragma unroll
        for (int i = 1; i < 4; ++i)
            if (a[i] > a[p0]) p0 = i;
        int p1 = p0 == 0 ? 1 : 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i != p0 && a[i] > a[p1]) p1 = i;
        const int i0 = min(p0, p1), i1 = max(p0, p1);
#pragma unroll
        for (int i = 0; i < 4; ++i) Wp[(k0 + i) * N + n] = (i == i0 || i == i1) ? v[i] : 0.0f;
        word |= (uint32_t)((i1 << 2) | i0) << (4 * b);
    }
    meta[(int64_t)kw * N + n] = word;
}

// One thread per (column, 16 rows = 4 blocks): one word of kept codes.
__global__ void __launch_bounds__(256) pack24_kernel(const uint8_t* __restrict__ codes,
                                                     const uint32_t* __restrict__ meta, int K, int N,
                                                     uint32_t* __restrict__ vals)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int vw = blockIdx.y;  // value word: rows 16 vw .. 16 vw + 15
    if (n >= N) return;
    const uint32_t m = __ldg(meta + (int64_t)(vw >> 1) * N + n);
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int b = 4 * vw + j;  // global block index
        const uint32_t nib = (m >> (4 * (b & 7))) & 0xFu;
        const int64_t k0 = 4 * (int64_t)b;
        const uint32_t c0 = __ldg(codes + (k0 + (nib & 3u)) * N + n) & 0xFu;
        const uint32_t c1 = __ldg(codes + (k0 + (nib >> 2)) * N + n) & 0xFu;
        word |= (c0 | (c1 << 4)) << (8 * j);
    }
    vals[(int64_t)vw * N + n] = word;
}

// The tensor-core layout of the kept codes (the mma.sp decode kernel's operand): per
// group of 128 rows (32 blocks) and column, word u = 2 t + hb (t = 0..3, hb = 0..1) holds,
// for the group's four 32-row steps s, the kept pair of block 8 s + t + 4 hb: its first
// kept code at bits 4 s, its second at bits 16 + 4 s.  vals_tc[8 gq + u][n]; one thread per
// (group, column) reads the group's 8 canonical words and writes its 8 words.
__global__ void __launch_bounds__(256) pack24_tc_kernel(const uint32_t* __restrict__ vals, int K, int N,
                                                        uint32_t* __restrict__ vals_tc)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int gq = blockIdx.y;
    if (n >= N) return;
    uint32_t v[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) v[w] = __ldg(vals + (int64_t)(8 * gq + w) * N + n);  // blocks 4w .. 4w + 3
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int t = u >> 1, hb = u & 1;
        uint32_t out = 0;
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const int bl = 8 * st + t + 4 * hb;
            const uint32_t byte = (v[bl >> 2] >> (8 * (bl & 3))) & 0xFFu;  // (second << 4) | first
            out |= (byte & 0xFu) << (4 * st);
            out |= (byte >> 4) << (16 + 4 * st);
        }
        vals_tc[(int64_t)(8 * gq + u) * N + n] = out;
    }
}

// Y[m][n] = rn(sum over kept k of X[m][k] * (q - z) * s): one thread per column and MT
// tokens; per group of 128 rows the thread reads its fp16 scale, zero, 8 value words and
// 4 metadata words (each coalesced along N) and gathers X from L1/L2.  (q - z) * s is
// exact in fp32 (a 5-bit integer times an 11-bit scale); the products are summed with
// fp32 fused multiply-adds in k order.  A SIMT kernel for the decode regime (few
// tokens), where the weight stream dominates.
template <int MT, bool BF16>
__global__ void __launch_bounds__(128) gemm_w4a16_24_kernel(const uint16_t* __restrict__ X, int M, int K, int N,
                                                            const uint32_t* __restrict__ vals,
                                                            const uint32_t* __restrict__ meta,
                                                            const uint16_t* __restrict__ scales,
                                                            const uint8_t* __restrict__ zeros, uint16_t* __restrict__ Y)
{
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int m0 = blockIdx.y * MT;
    if (n >= N) return;
    const int G = K / 128;
    float acc[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t] = 0.0f;
    for (int g = 0; g < G; ++g) {
        const float s = __half2float(__ushort_as_half(__ldg(scales + (int64_t)g * N + n)));
        const int z = (int)__ldg(zeros + (int64_t)g * N + n);
#pragma unroll 1
        for (int mw = 0; mw < 4; ++mw) {  // 4 metadata words = 32 blocks = 128 rows
            const uint32_t m = __ldg(meta + (int64_t)(4 * g + mw) * N + n);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // 2 value words per metadata word
                const uint32_t v = __ldg(vals + (int64_t)(8 * g + 2 * mw + h) * N + n);
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // 4 blocks per value word
                    const int bl = 4 * h + j;  // block inside the metadata word
                    const uint32_t nib = (m >> (4 * bl)) & 0xFu;
                    const int k0 = 128 * g + 32 * mw + 4 * bl;
                    const int ka = k0 + (int)(nib & 3u), kb = k0 + (int)(nib >> 2);
                    const float wa = (float)((int)((v >> (8 * j)) & 0xFu) - z) * s;
                    const float wb = (float)((int)((v >> (8 * j + 4)) & 0xFu) - z) * s;
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        if (m0 + t < M) {
                            const uint16_t* xr = X + (int64_t)(m0 + t) * K;
                            const float xa = BF16 ? bf16_bits_to_f32(__ldg(xr + ka)) : __half2float(__ushort_as_half(__ldg(xr + ka)));
                            const float xb = BF16 ? bf16_bits_to_f32(__ldg(xr + kb)) : __half2float(__ushort_as_half(__ldg(xr + kb)));
                            acc[t] = fmaf(xa, wa, acc[t]);
                            acc[t] = fmaf(xb, wb, acc[t]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t)
        if (m0 + t < M) Y[(int64_t)(m0 + t) * N + n] = BF16 ? f32_to_bf16_bits(acc[t]) : f32_to_f16_bits(acc[t]);
}

}  // namespace qg
