// w4a16_skinny.cuh -- decode-shape W4A16 fused dequant-GEMM (M <= 32).
//
// Computes Y = X * W_deq with W_deq[k][n] = (q[k][n] - z[g][n]) * s[g][n]
// ("AI Infra guide, ch.4 Quantization" sec. 3.1 weight-only INT4 and sec. 3.5 fused
// INT4 x FP16 kernel; per-group scale and zero: "LLM inference cost: W8A8/W4A8 ..."
// sec. 2.2).  At decode shapes the weight stream is the whole cost, so the kernel is
// built around reading packed INT4 words from HBM exactly once, at full width:
//
//  * Swap-AB on the tensor cores: the weight tile is the MMA's A operand (16 output
//    columns per m16 tile) and the few tokens are its N = 8 operand, so M = 1..32
//    wastes no weight bandwidth.  mma.sync keeps both operands in registers: the
//    dequantized weights never touch shared memory.
//  * Each lane issues one 128-bit load per 32 k x 4 columns (4 words, 8 k each); a
//    warp load covers 4 full 128-byte rows of the packed matrix.  A ring of
//    `DEPTH` steps of loads stays in flight per lane.
//  * The k order inside one 32-k step is permuted so that a lane's own word feeds
//    its fragment slots directly: slots (2t, 2t+1, 2t+8, 2t+9) of the two k16 MMAs
//    take nibbles (0,4,1,5) and (2,6,3,7) of word kb = 4*step + t.  The activation
//    fragment uses the same permutation (two byte-permutes per register pair).
//  * Dequantization is two packed half-precision ops per pair of weights: the
//    nibble pair is OR-ed into the exponent field (128 + q for bf16, 1024 + q for
//    fp16, both exact), (128 + z) is subtracted exactly, and one multiply by the
//    scale rounds once to the activation dtype.
//  * Split-K across a thread-block cluster along grid.y: every CTA reduces its warps'
//    fragments in shared memory, then each CTA of the cluster sums one slice of the
//    columns over all cluster ranks through distributed shared memory, in rank
//    order, and writes Y.  No global workspace, no atomics, deterministic.
#pragma once
#include "common.cuh"

namespace qg {

template <bool BF16>
struct HalfOps {
    static constexpr uint32_t MAGIC = BF16 ? 0x43004300u : 0x64006400u;  // 128.0 / 1024.0 in both halves
    static constexpr float BIAS = BF16 ? 128.0f : 1024.0f;
    QG_DEV_INLINE static uint32_t sub2(uint32_t a, uint32_t b)
    {
        uint32_t r;
        if constexpr (BF16) asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        return r;
    }
    QG_DEV_INLINE static uint32_t mul2(uint32_t a, uint32_t b)
    {
        uint32_t r;
        if constexpr (BF16) asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        else asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
        return r;
    }
    QG_DEV_INLINE static uint32_t splat(float v) { return BF16 ? pack_bf16x2_rn(v, v) : pack_f16x2_rn(v, v); }
    QG_DEV_INLINE static uint16_t to_bits(float v) { return BF16 ? f32_to_bf16_bits(v) : f32_to_f16_bits(v); }
};

// Sparse m16n8k32 (2:4 along k): a0..a3 hold the kept pairs of the compressed A
// (row g, block t | row g + 8, block t | row g, block t + 4 | row g + 8, block t + 4),
// b0..b3 the dense B rows 2t + 8i (+1), e the position nibbles (selector 0: lanes t = 0, 1).
template <bool BF16>
QG_DEV_INLINE void mma_sp_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                uint32_t b1, uint32_t b2, uint32_t b3, uint32_t e)
{
    if constexpr (BF16)
        asm("mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(b2), "r"(b3), "r"(e));
    else
        asm("mma.sp::ordered_metadata.sync.aligned.m16n8k32.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9,%10,%11}, {%0,%1,%2,%3}, %12, 0x0;"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(b2), "r"(b3), "r"(e));
}

template <bool BF16>
QG_DEV_INLINE void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                             uint32_t b1)
{
    if constexpr (BF16)
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct SkinnyParams {
    const uint16_t* X;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint8_t* zeros;
    uint16_t* Y;
    int M, K, N;
};

// MT: token tiles of 8 (M <= 8*MT).  WN: warps along N (64 columns each).
// WK: warps along K.  DEPTH: 32-k steps of weight loads kept in flight per lane.
template <int MT, bool BF16, int WN, int WK, int DEPTH>
__global__ void __launch_bounds__(WN* WK * 32, 1) w4a16_skinny_kernel(const SkinnyParams p)
{
    using H = HalfOps<BF16>;
    constexpr int BN = 64 * WN;
    constexpr int MP = 8 * MT;
    extern __shared__ __align__(16) float red[];  // [WK][BN][MP]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wn = warp % WN, wk = warp / WN;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int N = p.N, K = p.K, M = p.M;
    const int n0 = blockIdx.x * BN;
    const int nw = n0 + 64 * wn;

    // K range of this CTA (whole groups of 128), then this warp's contiguous steps
    const int S = gridDim.y;
    const int rank = blockIdx.y;
    const int G = K >> 7;
    const int g_lo = (int)((int64_t)G * rank / S), g_hi = (int)((int64_t)G * (rank + 1) / S);
    const int T = 4 * (g_hi - g_lo);
    const int s_lo = 4 * g_lo + (int)((int64_t)T * wk / WK);
    const int s_hi = 4 * g_lo + (int)((int64_t)T * (wk + 1) / WK);

    // column bases of this lane's two 128-bit words per step (4 columns each)
    int ncol[2];
    bool nval[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        ncol[h] = nw + 32 * h + 4 * g8;
        nval[h] = ncol[h] < N;
    }

    float acc[2][2][MT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][c][j][e] = 0.0f;

    uint4 buf[DEPTH][2];
    auto load_step = [&](int s, uint4 (&b)[2]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (s < s_hi && nval[h])
                b[h] = ldg_stream_v4(p.packed + (int64_t)(4 * s + t4) * N + ncol[h]);
            else
                b[h] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
#pragma unroll
    for (int i = 0; i < DEPTH; ++i) load_step(s_lo + i, buf[i]);

    // per-group dequant constants for the lane's 8 columns, prefetched one group ahead
    uint2 sc_next[2];
    uint32_t zr_next[2];
    auto load_group = [&](int g) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (g < g_hi && nval[h]) {
                sc_next[h] = __ldg(reinterpret_cast<const uint2*>(p.scales + (int64_t)g * N + ncol[h]));
                zr_next[h] = __ldg(reinterpret_cast<const uint32_t*>(p.zeros + (int64_t)g * N + ncol[h]));
            } else {
                sc_next[h] = make_uint2(0u, 0u);
                zr_next[h] = 0u;
            }
        }
    };
    uint32_t s2[2][4], zb2[2][4];
    int cur_g = -1;
    if (s_lo < s_hi) load_group(s_lo >> 2);

    const uint16_t* xbase = p.X;

#pragma unroll 1
    for (int base = s_lo; base < s_hi; base += DEPTH) {
#pragma unroll
        for (int i = 0; i < DEPTH; ++i) {
            const int s = base + i;
            if (s < s_hi) {
                const int g = s >> 2;
                if (g != cur_g) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t sw[2] = {sc_next[h].x, sc_next[h].y};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float sv = __half2float(__ushort_as_half((unsigned short)(sw[c >> 1] >> (16 * (c & 1)))));
                            const float zv = (float)((zr_next[h] >> (8 * c)) & 0xFFu);
                            s2[h][c] = H::splat(sv);
                            zb2[h][c] = H::splat(H::BIAS + zv);
                        }
                    }
                    cur_g = g;
                    load_group(g + 1);
                }
                // activation fragments: X[token][8*kb .. 8*kb+7], kb = 4s + t, permuted (0,4)(1,5)(2,6)(3,7)
                uint32_t xb[MT][4];
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const int tok = 8 * j + g8;
                    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                    if (tok < M) xv = ldg_v4(xbase + (int64_t)tok * K + 8 * (4 * s + t4));
                    xb[j][0] = prmt(xv.x, xv.z, 0x5410);
                    xb[j][1] = prmt(xv.x, xv.z, 0x7632);
                    xb[j][2] = prmt(xv.y, xv.w, 0x5410);
                    xb[j][3] = prmt(xv.y, xv.w, 0x7632);
                }
                // dequantize the lane's 8 words: R[h][c][r] = (nib r, nib r+4) of word (h, c)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w[4] = {buf[i][h].x, buf[i][h].y, buf[i][h].z, buf[i][h].w};
                    uint32_t R[4][4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const uint32_t v = lop3_and_or(w[c] >> (4 * r), 0x000F000Fu, H::MAGIC);
                            R[c][r] = H::mul2(H::sub2(v, zb2[h][c]), s2[h][c]);
                        }
                    }
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            mma_16816<BF16>(acc[h][cp][j], R[2 * cp][0], R[2 * cp + 1][0], R[2 * cp][1],
                                            R[2 * cp + 1][1], xb[j][0], xb[j][1]);
                            mma_16816<BF16>(acc[h][cp][j], R[2 * cp][2], R[2 * cp + 1][2], R[2 * cp][3],
                                            R[2 * cp + 1][3], xb[j][2], xb[j][3]);
                        }
                }
                load_step(s + DEPTH, buf[i]);
            }
        }
    }

    // ---- reduction 1: warps along K, in shared memory ----
    float* myred = red + (size_t)wk * BN * MP;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int cp = 0; cp < 2; ++cp)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                const int nl = 64 * wn + 32 * h + 4 * g8 + 2 * cp;
                const int tk = 8 * j + 2 * t4;
                *reinterpret_cast<float2*>(myred + (size_t)nl * MP + tk) = make_float2(acc[h][cp][j][0], acc[h][cp][j][1]);
                *reinterpret_cast<float2*>(myred + (size_t)(nl + 1) * MP + tk) =
                    make_float2(acc[h][cp][j][2], acc[h][cp][j][3]);
            }
    __syncthreads();
    for (int e = threadIdx.x; e < BN * MP; e += blockDim.x) {
        float v = red[e];
#pragma unroll
        for (int q = 1; q < WK; ++q) v += red[(size_t)q * BN * MP + e];
        red[e] = v;
    }
    // ---- reduction 2: CTAs of the cluster (split-K), through distributed shared memory ----
    cluster_sync();
    const int slice = BN / S;
    const int c0 = rank * slice;
    const uint32_t red_s = smem_u32(red);
    for (int e = threadIdx.x; e < slice * M; e += blockDim.x) {
        const int tok = e / slice, nn = c0 + e % slice;
        const int n = n0 + nn;
        float v = 0.0f;
        const uint32_t off = (uint32_t)((nn * MP + tok) * 4);
        for (int q = 0; q < S; ++q) v += ld_dsmem_f32(dsmem_addr(red_s + off, q));
        if (n < N) p.Y[(int64_t)tok * N + n] = H::to_bits(v);
    }
    cluster_sync();
}

}  // namespace qg
