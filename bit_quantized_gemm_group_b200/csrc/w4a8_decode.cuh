// w4a8_decode.cuh -- W4A8 GEMM for token counts up to 64 per launch, on the tcgen05
// tensor cores.
//
//   P[m][g][n] = sum_{k in group g} Xq[m][k] q[k][n]          (int32, exact)
//   Y[m][n]    = bf16_rn( t[m] * sum_g float(P[m][g][n]) sg[g][n] )   (fp32)
// ("LLM inference cost: W8A8/W4A8 ..." sec. 2.2: INT4 weights in groups of 128 with a
// per-group scale, INT8 activations with a per-token scale.)  At these M the product
// streams the packed weights once: HBM-bound.
//
// Stream-K over (128-column slab, group) units, as in the W8A8 and W4A16 decode
// kernels.  Swap-AB: the 128 columns are the MMA's M, the tokens its N (16/32/64).
//   * TMA brings a unit's packed words (16 rows x 128 columns) and token tile.
//   * Dequant warps (thread = column and k-half) sign-extend the nibbles to int8 and store
//     the unit's 128 x 128 weight tile into one of AS tensor-memory A buffers (lane =
//     column, four consecutive k per 32-bit column), the MMA's A operand: no shared-memory
//     round trip and no generic-to-async proxy fence on the way.
//   * NI threads, each in a warp of its own, issue the MMAs (units i = e mod NI), one
//     group's P into a TMEM buffer of their own: an MMA holds its issuing thread for a
//     while, and a unit here is half the bytes of a W8A8 unit.
//   * Epilogue warps (thread = column) read each group's P, add float(P) s_g into fp32
//     registers (and, on request, store P), and at a piece end finish Y, or publish the
//     fp32 piece in the workspace under the launch's token (a split slab's later pieces,
//     always their CTAs' first), or, holding the slab's first group (always the CTA's
//     last piece), wait (bounded) for the other pieces' tokens, add them in CTA order and
//     finish Y.  One launch per call.
// Stage ring, A buffers and D buffers have even depth, so every mbarrier has one consumer
// that waits on its phases in order.
#pragma once
#include "common.cuh"
#include "int8_decode.cuh"

namespace qg {

struct W4A8DecodeParams {
    const float* t;    // fp32 [M]
    const float* sg;   // fp32 [G][N]
    uint16_t* Y;       // bf16 [M][N]
    int32_t* dbg;      // NULL or int32 [M][G][N]: receives every P
    float* partials;   // [grid][NT][128]: the CTA's published piece
    unsigned long long* flags;  // [grid] publication tokens
    unsigned long long token;   // this launch's token (never 0)
    int M, K, N;
    int G, nslabs, units, grid;
};

template <int NT, int NI_>
struct W4A8DecCfg {
    static constexpr int X_BYTES = NT * 128;       // NT tokens x 128 k (int8), 128-byte swizzle
    static constexpr int RAW_BYTES = 16 * 128 * 4;  // packed words: 16 rows x 128 columns
    static constexpr int STAGE = (X_BYTES + RAW_BYTES + 1023) / 1024 * 1024;
    static constexpr int NI = NI_;
    static_assert(NI == 2 || NI == 4, "issuer count divides the ring depths");
    // ring depths, multiples of NI so that stage s / A buffer a always feeds issuer s % NI
    static constexpr int ST = 8;
    static constexpr int AS = 8;
    static constexpr int EARLY = 4;
    // tensor memory: D buffers [NI][DP] of NT columns, then AS A buffers of 32 columns
    static constexpr int DP = NI * 4 * NT + AS * 32 <= 512 ? 4 : 2;
    static constexpr int A_COL0 = NI * DP * NT;
    static constexpr int TMEM_NEED = A_COL0 + AS * 32;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "tensor memory budget");
    static constexpr int DQ = 8;                   // dequant warps: 4 lane quarters x 2 k-halves
    static constexpr int EH = NT >= 64 ? 2 : 1;     // epilogue warps per lane quarter
    static constexpr int EPI = 4 * EH;
    static constexpr int TPW = NT / EH;             // tokens of one epilogue thread
    // warp 0 producer; issuers in warps 1..3 and then after the dequant warps;
    // epilogue warps 4 .. 4+EPI-1; dequant warps DQ0 .. DQ0+7
    static constexpr int DQ0 = 4 + EPI;
    static constexpr int XI0 = DQ0 + DQ;            // issuer 3 onwards
    static constexpr int THREADS = 32 * (XI0 + (NI > 3 ? NI - 3 : 0));
    static constexpr int BAR_OFF = ST * STAGE;
    // full[ST] empty[ST] afull[AS] aempty[AS] dfull[NI][DP] dempty[NI][DP] done[NI]
    static constexpr int NBAR = 2 * ST + 2 * AS + 2 * NI * DP + NI;
    static constexpr int T_OFF = BAR_OFF + NBAR * 8 + 16;  // token scales t[0..NT)
    static constexpr int LA = 8;                          // group scales fetched LA units ahead
    static constexpr int SG_OFF = T_OFF + NT * 4;         // [EPI][LA][32] fp32 ring
    static constexpr int TOTAL = SG_OFF + EPI * LA * 32 * 4 + 1024;
    // empty[s]: the dequant warps (packed words read) and the MMA commit (token tile read)
    static constexpr uint32_t EMPTY_ARRIVALS = DQ + 1;
};

template <int NT, int NI>
__global__ void __launch_bounds__(W4A8DecCfg<NT, NI>::THREADS, 1)
    w4a8_decode_kernel(const W4A8DecodeParams p, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_x)
{
    using C = W4A8DecCfg<NT, NI>;
    constexpr int ST = C::ST, AS = C::AS, DP = C::DP;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + ST;
    uint64_t* afull = empty + ST;
    uint64_t* aempty = afull + AS;
    uint64_t* dfull = aempty + AS;          // [NI][DP]
    uint64_t* dempty = dfull + C::NI * DP;  // [NI][DP]
    uint64_t* done = dempty + C::NI * DP;   // [NI]
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + C::NI);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;
    const int u0 = i8_first_unit(blockIdx.x, p.units, p.grid), u1 = i8_first_unit(blockIdx.x + 1, p.units, p.grid);
    const int n_it = u1 - u0;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], C::EMPTY_ARRIVALS);
        }
        for (int i = 0; i < AS; ++i) {
            mbar_init(&afull[i], C::DQ);
            mbar_init(&aempty[i], 1);
        }
        for (int i = 0; i < C::NI * DP; ++i) {
            mbar_init(&dfull[i], 1);
            mbar_init(&dempty[i], 32 * C::EPI);
        }
        for (int i = 0; i < C::NI; ++i) mbar_init(&done[i], 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tslot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;

    if (warp == 0) {
        // ---------------- producer: one thread issues TMA ----------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_w);
            tma_prefetch_desc(&tm_x);
            // packed words do not depend on the previous grid: the first EARLY stages of
            // them are requested before waiting for it; the token tiles after
            int i = 0;
            bool waited = false;
            for (; i < n_it; ++i) {
                const int u = u0 + i, s = i % ST;
                if (!mbar_wait(&empty[s], ((i / ST) & 1) ^ 1)) break;
                uint8_t* st = smem + s * C::STAGE;
                const int slab = u / G, g = u % G;
                mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::RAW_BYTES);
                tma_load_2d(&tm_w, &full[s], st + C::X_BYTES, slab * 128, 16 * g);
                if (waited) {
                    tma_load_2d(&tm_x, &full[s], st, g * 128, 0);
                } else if (i + 1 == C::EARLY || i + 1 == n_it) {
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    waited = true;
                    for (int j = 0; j <= i; ++j)
                        tma_load_2d(&tm_x, &full[j % ST], smem + (j % ST) * C::STAGE, ((u0 + j) % G) * 128, 0);
                }
            }
            if (!waited) {  // gave up inside the first stages: complete them so that they can land
                asm volatile("griddepcontrol.wait;" ::: "memory");
                for (int j = 0; j < i; ++j)
                    tma_load_2d(&tm_x, &full[j % ST], smem + (j % ST) * C::STAGE, ((u0 + j) % G) * 128, 0);
            }
            for (int j = i - ST > 0 ? i - ST : 0; j < i; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        }
    } else if ((warp >= 1 && warp <= 3 && warp <= NI) || warp >= C::XI0) {
        // ---------------- MMA issuers: units i = e (mod NI), one group each ----------------
        if (lane == 0) {
            const int e = warp <= 3 ? warp - 1 : 3 + warp - C::XI0;
            constexpr uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                                       ((uint32_t)(128 >> 4) << 24);  // s32 += s8 x s8, both K-major
            bool issued = false;
            for (int i = e; i < n_it; i += NI) {
                const int j = i / NI, d = e * DP + j % DP, s = i % ST, a = i % AS;
                if (!mbar_wait(&dempty[d], ((j / DP) & 1) ^ 1)) break;
                if (!mbar_wait(&full[s], (i / ST) & 1)) break;
                if (!mbar_wait(&afull[a], (i / AS) & 1)) break;
                tc_fence_after();
                const uint32_t xs = smem_u32(smem + s * C::STAGE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 32 k = 8 A columns per step
                    mma_i8_ts(tmem + d * NT, tmem + C::A_COL0 + 32 * a + 8 * kk, smem_desc(xs + 32 * kk, 16, 1024, 2),
                              idesc, kk > 0 ? 1u : 0u);
                mma_commit(&aempty[a]);
                mma_commit(&empty[s]);
                mma_commit(&dfull[d]);
                issued = true;
            }
            if (issued) {  // every MMA has completed before tensor memory is released
                mma_commit(&done[e]);
                mbar_wait(&done[e], 0);
            }
        }
    } else if (warp >= 4 && warp < C::DQ0) {
        // ---------------- epilogue: one thread per column and token range ----------------
        asm volatile("griddepcontrol.wait;" ::: "memory");  // t, sg, Y and the workspace follow the previous grid
        constexpr int TPW = C::TPW;
        const int q = warp & 3, col = 32 * q + lane;
        const int tb = ((warp - 4) >> 2) * TPW;  // first token of this warp
        const int M = p.M;
        float* ts = reinterpret_cast<float*>(smem + C::T_OFF);
        for (int t = threadIdx.x - 128; t < M; t += 32 * C::EPI) ts[t] = __ldg(p.t + t);
        named_bar_sync(1, 32 * C::EPI);
        // s_g of this thread's column for unit i lands in ring slot i % LA, LA units ahead
        // of its use, so no global load latency sits on the unit loop
        constexpr int LA = C::LA;
        float* sgr = reinterpret_cast<float*>(smem + C::SG_OFF) + (warp - 4) * LA * 32 + lane;
        auto fetch_sg = [&](int i) {
            if (i < n_it) {
                const int u = u0 + i, n = (u / G) * 128 + col;
                cp_async_4(sgr + (i % LA) * 32, p.sg + (n < p.N ? (int64_t)(u % G) * p.N + n : 0), n < p.N);
            }
            cp_async_commit();  // one group per unit, empty past the end
        };
#pragma unroll
        for (int i = 0; i < LA - 1; ++i) fetch_sg(i);
        const int64_t dstride = (int64_t)G * p.N;  // token stride of the debug output
        float acc[TPW];
#pragma unroll
        for (int t = 0; t < TPW; ++t) acc[t] = 0.f;
        bool ok = true;  // after a wait gives up, the units are still walked (named barriers) without work
        for (int i = 0; i < n_it; ++i) {
            const int u = u0 + i, slab = u / G, g = u % G, n = slab * 128 + col;
            const int e = i % NI, j = i / NI, d = e * DP + j % DP;
            fetch_sg(i + LA - 1);
            cp_async_wait_group<LA - 1>();  // unit i's group has landed
            const float sv = sgr[(i % LA) * 32];
            if (ok && !mbar_wait(&dfull[d], (j / DP) & 1)) ok = false;
            if (ok) {
            tc_fence_after();
            const uint32_t dcol = tmem + ((uint32_t)(32 * q) << 16) + d * NT + tb;
#pragma unroll
            for (int t0 = 0; t0 < TPW; t0 += 16) {
                if (tb + t0 < M) {
                    uint32_t P[16];
                    tmem_ld_32x32b_x16(dcol + t0, P);
                    tmem_ld_wait();
#pragma unroll
                    for (int t = 0; t < 16; ++t) acc[t0 + t] = fmaf(i2f_small(P[t]), sv, acc[t0 + t]);  // |P| < 2^17
                }
            }
            if (p.dbg) {  // the exact P, on request: one column at a time, off the fast path
                int32_t* dbg = p.dbg + (int64_t)g * p.N + n + tb * dstride;
#pragma unroll 1
                for (int t = 0; t < TPW && tb + t < M; ++t) {
                    const uint32_t v = tmem_ld_32x32b_x1(dcol + t);
                    tmem_ld_wait();
                    if (n < p.N) dbg[t * dstride] = (int32_t)v;
                }
            }
            tc_fence_before();
            mbar_arrive(&dempty[d]);
            }
            if (i + 1 == n_it || g == G - 1) {
                // piece end: a whole slab finishes Y; a later piece of a split slab is
                // published; the piece holding the slab's first group finishes the slab
                const int gstart = slab == u0 / G ? u0 % G : 0;
                const bool whole = gstart == 0 && g == G - 1;
                const bool head = gstart == 0 && !whole;
                if (head) {
                    const int cl = i8_cta_of_unit(slab * G + G - 1, p.units, p.grid);
                    bool ready = true;
                    if (warp == 4 && ok) ready = watch_tokens(p.flags, (int)blockIdx.x + 1, cl, p.token, lane);
                    if (!named_bar_and(1, 32 * C::EPI, ok && ready)) ok = false;
                    if (ok) {
                        // the other pieces in CTA order (the order of the sum is fixed)
                        for (int c = (int)blockIdx.x + 1; c <= cl; ++c) {
                            const float* other = p.partials + (size_t)c * NT * 128 + tb * 128 + col;
#pragma unroll
                            for (int t = 0; t < TPW; ++t)
                                if (tb + t < M) acc[t] += __ldcg(other + t * 128);
                        }
                    }
                }
                if (whole || head) {
                    if (ok && n < p.N) {
                        uint16_t* y = p.Y + (int64_t)tb * p.N + n;
#pragma unroll
                        for (int t = 0; t < TPW; ++t)
                            if (tb + t < M) y[(int64_t)t * p.N] = f32_to_bf16_bits(__fmul_rn(ts[tb + t], acc[t]));
                    }
                } else {
                    float* mine = p.partials + (size_t)blockIdx.x * NT * 128 + tb * 128 + col;
                    if (ok) {
#pragma unroll
                        for (int t = 0; t < TPW; ++t)
                            if (tb + t < M) __stcg(mine + t * 128, acc[t]);
                    }
                    // publish: every epilogue thread's stores, then one fence and the token
                    named_bar_sync(1, 32 * C::EPI);
                    if (ok && threadIdx.x == 128) {
                        __threadfence();
                        st_release_u64(p.flags + blockIdx.x, p.token);
                    }
                }
#pragma unroll
                for (int t = 0; t < TPW; ++t) acc[t] = 0.f;
            }
        }
        cp_async_wait_group<0>();  // no copy into shared memory outlives the loop
    } else if (warp >= C::DQ0 && warp < C::XI0) {
        // ---------------- dequant: packed words -> int8 weight tile in tensor memory ----------------
        static_assert(C::DQ0 % 4 == 0, "a dequant warp stores to the lane quarter warp % 4");
        const int q = (warp - C::DQ0) & 3, kh = (warp - C::DQ0) >> 2;  // lane quarter, k-half
        const int col = 32 * q + lane;
        for (int i = 0; i < n_it; ++i) {
            const int s = i % ST, a = i % AS;
            if (!mbar_wait(&full[s], (i / ST) & 1)) break;
            const uint32_t* raw = reinterpret_cast<const uint32_t*>(smem + s * C::STAGE + C::X_BYTES);
            uint32_t w[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) w[r] = raw[(8 * kh + r) * 128 + col];
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);  // packed words consumed
            uint32_t o[16];  // k = 4r .. 4r+3 of this k-half in o[r]
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 16 k = two words
#pragma unroll
                for (int hw = 0; hw < 2; ++hw) {
                    // nibbles -> bytes (even k, odd k), sign-extended from 4 bits, then
                    // interleaved back into k order
                    const uint32_t word = w[2 * c + hw];
                    uint32_t ev, od;
                    asm("lop3.b32 %0, %1, 0x0F0F0F0F, 0x08080808, 0x6A;" : "=r"(ev) : "r"(word));
                    asm("lop3.b32 %0, %1, 0x0F0F0F0F, 0x08080808, 0x6A;" : "=r"(od) : "r"(word >> 4));
                    ev = (ev + 0x78787878u) ^ 0x80808080u;
                    od = (od + 0x78787878u) ^ 0x80808080u;
                    o[4 * c + 2 * hw] = prmt(ev, od, 0x5140);
                    o[4 * c + 2 * hw + 1] = prmt(ev, od, 0x7362);
                }
            }
            if (!mbar_wait(&aempty[a], ((i / AS) & 1) ^ 1)) break;
            tc_fence_after();
            tmem_st_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + C::A_COL0 + 32 * a + 16 * kh, o);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace qg
