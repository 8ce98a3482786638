// int8_skinny.cuh -- decode-shape W8A8 and W4A8 GEMMs on int8 tensor cores.
//
// W8A8 (SmoothQuant, "AI Infra guide, ch.4 Quantization" sec. 2.2-2.3):
//     acc = sum_k Xq[m][k] Wq[k][n] (int32, exact);  Y = bf16(((float)acc * t[m]) * sw[n])
// W4A8 (group-wise 4-bit weights with 8-bit activations, "LLM inference cost:
// W8A8/W4A8 ..." sec. 2.2):
//     P[m][g][n] = sum_{k in g} Xq[m][k] q[k][n] (int32);  Y = bf16(t[m] * sum_g P * sg[g][n])
//
// Same decode design as the W4A16 kernel: swap-AB mma.sync (weights are the
// m16 operand, up to 32 tokens are n8 tiles), weights read once from HBM with
// 128-bit streaming loads into registers, K split over warps and over a thread
// block cluster, reduced in shared and distributed shared memory.
//
// W8A8 weights are row-major int8 [K][N]: a lane loads 16 adjacent columns of 8
// consecutive k rows and transposes 4x4 byte blocks with byte permutes, so each
// register holds 4 k values of one column, as the int8 A fragment wants.
// W4A8 weights are packed 8 nibbles per word along K: the even and odd nibbles of a
// word are sign-extended to bytes in three integer ops per 4 values, and the
// activation bytes are permuted the same way (k order inside a step is free).
#pragma once
#include "common.cuh"

namespace qg {

QG_DEV_INLINE void mma_16832_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                uint32_t b1)
{
    asm(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4x4 byte transpose: out[j] = (a.byte j, b.byte j, c.byte j, d.byte j)
QG_DEV_INLINE void transpose4x4_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t (&o)[4])
{
    const uint32_t ab_lo = prmt(a, b, 0x5140), ab_hi = prmt(a, b, 0x7362);
    const uint32_t cd_lo = prmt(c, d, 0x5140), cd_hi = prmt(c, d, 0x7362);
    o[0] = prmt(ab_lo, cd_lo, 0x5410);
    o[1] = prmt(ab_lo, cd_lo, 0x7632);
    o[2] = prmt(ab_hi, cd_hi, 0x5410);
    o[3] = prmt(ab_hi, cd_hi, 0x7632);
}

// low nibbles of the 4 bytes of x (each in 0..15 as a two's-complement 4-bit value)
// -> 4 sign-extended int8 bytes.  u = nib ^ 8 lies in 0..15; (u + 0x78) ^ 0x80 = u - 8
// per byte, and no byte carries into its neighbour.
QG_DEV_INLINE uint32_t sext_nibbles_to_bytes(uint32_t x)
{
    uint32_t u;
    asm("lop3.b32 %0, %1, 0x0F0F0F0F, 0x08080808, 0x6A;" : "=r"(u) : "r"(x));  // (x & m) ^ c
    return (u + 0x78787878u) ^ 0x80808080u;
}

struct Int8SkinnyParams {
    const int8_t* Xq;
    const float* t;
    const int8_t* Wq;        // W8A8
    const float* sw;         // W8A8
    const uint32_t* packed;  // W4A8
    const float* sg;         // W4A8
    uint16_t* Y;
    int32_t* dbg;            // acc [M][N] (W8A8) or part [M][K/128][N] (W4A8), may be NULL
    int M, K, N;
};

// ---------------------------------------------------------------------------
// W8A8.  Warp tile: 128 columns x 32 k per step; a lane holds 16 columns x 8 rows.
// Tile i (0..7) of the warp: row g <-> column nw + 16g + 2i, row g+8 <-> +1.
// Lane (g, t) owns k rows k0 + 8t .. k0 + 8t + 7 of the step; slots 4t..4t+3 take
// rows 0..3 and slots 4t+16..4t+19 take rows 4..7.
// ---------------------------------------------------------------------------
template <int MT, int WN, int WK>
__global__ void __launch_bounds__(WN* WK * 32, 1) w8a8_skinny_kernel(const Int8SkinnyParams p)
{
    constexpr int BN = 128 * WN;
    constexpr int MP = 8 * MT;
    extern __shared__ __align__(16) int ired[];  // [WK][BN][MP]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wn = warp % WN, wk = warp / WN;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int N = p.N, K = p.K, M = p.M;
    const int n0 = blockIdx.x * BN;
    const int ncol = n0 + 128 * wn + 16 * g8;
    const bool nval = ncol < N;

    const int S = gridDim.y, rank = blockIdx.y;
    const int G = K >> 7;
    const int g_lo = (int)((int64_t)G * rank / S), g_hi = (int)((int64_t)G * (rank + 1) / S);
    const int T = 4 * (g_hi - g_lo);
    const int s_lo = 4 * g_lo + (int)((int64_t)T * wk / WK);
    const int s_hi = 4 * g_lo + (int)((int64_t)T * (wk + 1) / WK);

    int acc[8][MT][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0;

    uint4 cur[8], nxt[8];
    auto load_step = [&](int s, uint4 (&b)[8]) {
#pragma unroll
        for (int r = 0; r < 8; ++r)
            b[r] = (s < s_hi && nval) ? ldg_stream_v4(p.Wq + (int64_t)(32 * s + 8 * t4 + r) * N + ncol)
                                      : make_uint4(0u, 0u, 0u, 0u);
    };
    load_step(s_lo, cur);
#pragma unroll 1
    for (int s = s_lo; s < s_hi; ++s) {
        load_step(s + 1, nxt);
        uint32_t xb[MT][2];
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int tok = 8 * j + g8;
            uint2 xv = make_uint2(0u, 0u);
            if (tok < M) xv = __ldg(reinterpret_cast<const uint2*>(p.Xq + (int64_t)tok * K + 32 * s + 8 * t4));
            xb[j][0] = xv.x;
            xb[j][1] = xv.y;
        }
        // rows 0..3 -> slots 4t..4t+3 ; rows 4..7 -> slots 4t+16..4t+19
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            uint32_t lo[4], hi[4];
            const uint32_t* r32[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) r32[r] = reinterpret_cast<const uint32_t*>(&cur[r]);
            transpose4x4_bytes(r32[0][wi], r32[1][wi], r32[2][wi], r32[3][wi], lo);
            transpose4x4_bytes(r32[4][wi], r32[5][wi], r32[6][wi], r32[7][wi], hi);
            // lo[c] / hi[c] hold column offset 4*wi + c: tile 2*wi (c = 0, 1), tile 2*wi + 1 (c = 2, 3)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                mma_16832_s8(acc[2 * wi][j], lo[0], lo[1], hi[0], hi[1], xb[j][0], xb[j][1]);
                mma_16832_s8(acc[2 * wi + 1][j], lo[2], lo[3], hi[2], hi[3], xb[j][0], xb[j][1]);
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) cur[r] = nxt[r];
    }

    int* myred = ired + (size_t)wk * BN * MP;
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < MT; ++j) {
            const int nl = 128 * wn + 16 * g8 + 2 * i;
            const int tk = 8 * j + 2 * t4;
            *reinterpret_cast<int2*>(myred + (size_t)nl * MP + tk) = make_int2(acc[i][j][0], acc[i][j][1]);
            *reinterpret_cast<int2*>(myred + (size_t)(nl + 1) * MP + tk) = make_int2(acc[i][j][2], acc[i][j][3]);
        }
    __syncthreads();
    for (int e = threadIdx.x; e < BN * MP; e += blockDim.x) {
        int v = ired[e];
#pragma unroll
        for (int q = 1; q < WK; ++q) v += ired[(size_t)q * BN * MP + e];
        ired[e] = v;
    }
    cluster_sync();
    const int slice = BN / S, c0 = rank * slice;
    const uint32_t red_s = smem_u32(ired);
    for (int e = threadIdx.x; e < slice * M; e += blockDim.x) {
        const int tok = e / slice, nn = c0 + e % slice, n = n0 + nn;
        int v = 0;
        const uint32_t off = (uint32_t)((nn * MP + tok) * 4);
        for (int q = 0; q < S; ++q) v += __float_as_int(ld_dsmem_f32(dsmem_addr(red_s + off, q)));
        if (n < N) {
            const float y = __fmul_rn(__fmul_rn(__int2float_rn(v), __ldg(p.t + tok)), __ldg(p.sw + n));
            p.Y[(int64_t)tok * N + n] = f32_to_bf16_bits(y);
            if (p.dbg) p.dbg[(int64_t)tok * N + n] = v;
        }
    }
    cluster_sync();
}

// ---------------------------------------------------------------------------
// W4A8.  Same lane/column mapping as the W4A16 kernel: per step (32 k) a lane loads
// two uint4 of 4 words (4 columns x 8 k); word (h, c) of the lane is column
// nw + 32h + 4g + c.  Tile (h, cp): row g <-> word (h, 2cp), row g+8 <-> (h, 2cp+1).
// Slots 4t..4t+3 take the even nibbles (k = 0,2,4,6 of the word), slots
// 4t+16..4t+19 the odd ones.  Warps split whole groups, so every group's int32
// partial lives in one warp and is rescaled there.
// ---------------------------------------------------------------------------
template <int MT, int WN, int WK>
__global__ void __launch_bounds__(WN* WK * 32, 1) w4a8_skinny_kernel(const Int8SkinnyParams p)
{
    constexpr int BN = 64 * WN;
    constexpr int MP = 8 * MT;
    extern __shared__ __align__(16) float fred[];  // [WK][BN][MP]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wn = warp % WN, wk = warp / WN;
    const int g8 = lane >> 2, t4 = lane & 3;
    const int N = p.N, K = p.K, M = p.M;
    const int n0 = blockIdx.x * BN;
    const int nw = n0 + 64 * wn;
    const int S = gridDim.y, rank = blockIdx.y;
    const int G = K >> 7;
    const int cg_lo = (int)((int64_t)G * rank / S), cg_hi = (int)((int64_t)G * (rank + 1) / S);
    const int NG = cg_hi - cg_lo;
    const int g_lo = cg_lo + (int)((int64_t)NG * wk / WK), g_hi = cg_lo + (int)((int64_t)NG * (wk + 1) / WK);

    int ncol[2];
    bool nval[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        ncol[h] = nw + 32 * h + 4 * g8;
        nval[h] = ncol[h] < N;
    }
    float accf[2][2][MT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) accf[h][c][j][e] = 0.0f;

    const int s_lo = 4 * g_lo, s_hi = 4 * g_hi;
    uint4 cur[2], nxt[2];
    auto load_step = [&](int s, uint4 (&b)[2]) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
            b[h] = (s < s_hi && nval[h]) ? ldg_stream_v4(p.packed + (int64_t)(4 * s + t4) * N + ncol[h])
                                         : make_uint4(0u, 0u, 0u, 0u);
    };
    load_step(s_lo, cur);
#pragma unroll 1
    for (int g = g_lo; g < g_hi; ++g) {
        int P[2][2][MT][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int j = 0; j < MT; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) P[h][c][j][e] = 0;
        float4 sc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
            sc[h] = nval[h] ? __ldg(reinterpret_cast<const float4*>(p.sg + (int64_t)g * N + ncol[h]))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            const int s = 4 * g + st;
            load_step(s + 1, nxt);
            uint32_t xb[MT][2];
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                const int tok = 8 * j + g8;
                uint2 xv = make_uint2(0u, 0u);
                if (tok < M) xv = __ldg(reinterpret_cast<const uint2*>(p.Xq + (int64_t)tok * K + 32 * s + 8 * t4));
                xb[j][0] = prmt(xv.x, xv.y, 0x6420);  // bytes k = 0, 2, 4, 6
                xb[j][1] = prmt(xv.x, xv.y, 0x7531);  // bytes k = 1, 3, 5, 7
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w[4] = {cur[h].x, cur[h].y, cur[h].z, cur[h].w};
                uint32_t ev[4], od[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ev[c] = sext_nibbles_to_bytes(w[c]);
                    od[c] = sext_nibbles_to_bytes(w[c] >> 4);
                }
#pragma unroll
                for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        mma_16832_s8(P[h][cp][j], ev[2 * cp], ev[2 * cp + 1], od[2 * cp], od[2 * cp + 1], xb[j][0],
                                     xb[j][1]);
            }
            cur[0] = nxt[0];
            cur[1] = nxt[1];
        }
        // group done: rescale in fp32, optional exact partial dump
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float scv[4] = {sc[h].x, sc[h].y, sc[h].z, sc[h].w};
#pragma unroll
            for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const float s_r0 = scv[2 * cp], s_r1 = scv[2 * cp + 1];
                    accf[h][cp][j][0] = fmaf(i2f_small((uint32_t)P[h][cp][j][0]), s_r0, accf[h][cp][j][0]);
                    accf[h][cp][j][1] = fmaf(i2f_small((uint32_t)P[h][cp][j][1]), s_r0, accf[h][cp][j][1]);
                    accf[h][cp][j][2] = fmaf(i2f_small((uint32_t)P[h][cp][j][2]), s_r1, accf[h][cp][j][2]);
                    accf[h][cp][j][3] = fmaf(i2f_small((uint32_t)P[h][cp][j][3]), s_r1, accf[h][cp][j][3]);
                    if (p.dbg && nval[h]) {
                        const int n_r0 = ncol[h] + 2 * cp, tk = 8 * j + 2 * t4;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int tok = tk + (e & 1), n = n_r0 + (e >> 1);
                            if (tok < M) p.dbg[((int64_t)tok * G + g) * N + n] = P[h][cp][j][e];
                        }
                    }
                }
        }
    }

    float* myred = fred + (size_t)wk * BN * MP;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int cp = 0; cp < 2; ++cp)
#pragma unroll
            for (int j = 0; j < MT; ++j) {
                const int nl = 64 * wn + 32 * h + 4 * g8 + 2 * cp;
                const int tk = 8 * j + 2 * t4;
                *reinterpret_cast<float2*>(myred + (size_t)nl * MP + tk) = make_float2(accf[h][cp][j][0], accf[h][cp][j][1]);
                *reinterpret_cast<float2*>(myred + (size_t)(nl + 1) * MP + tk) =
                    make_float2(accf[h][cp][j][2], accf[h][cp][j][3]);
            }
    __syncthreads();
    for (int e = threadIdx.x; e < BN * MP; e += blockDim.x) {
        float v = fred[e];
#pragma unroll
        for (int q = 1; q < WK; ++q) v += fred[(size_t)q * BN * MP + e];
        fred[e] = v;
    }
    cluster_sync();
    const int slice = BN / S, c0 = rank * slice;
    const uint32_t red_s = smem_u32(fred);
    for (int e = threadIdx.x; e < slice * M; e += blockDim.x) {
        const int tok = e / slice, nn = c0 + e % slice, n = n0 + nn;
        float v = 0.0f;
        const uint32_t off = (uint32_t)((nn * MP + tok) * 4);
        for (int q = 0; q < S; ++q) v += ld_dsmem_f32(dsmem_addr(red_s + off, q));
        if (n < N) p.Y[(int64_t)tok * N + n] = f32_to_bf16_bits(__fmul_rn(__ldg(p.t + tok), v));
    }
    cluster_sync();
}

}  // namespace qg
