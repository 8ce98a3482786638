// int8_decode.cuh -- W8A8 GEMM for token counts below the tile kernels' (M < 128), on
// the tcgen05 tensor cores.
//
//   acc[m][n] = sum_k Xq[m][k] Wq[k][n]     (int32, exact)
//   Y[m][n]   = bf16_rn( (float(acc) * t[m]) * sw[n] )
// ("AI Infra guide, ch.4 Quantization" sec. 2.2-2.3: SmoothQuant W8A8 with per-token
// dynamic activation scales and per-channel weight scales.)  At these M the product
// streams the int8 weights once: HBM-bound.
//
// Swap-AB.  The 128 columns of a slab are the MMA's M; the tokens are its N (16, 32, 64
// or 128, rows past M are zero).  A = the weight tile straight from Wq[K][N] (TMA box of
// 128 columns x 128 k, 128-byte swizzle), read by the MMA as an MN-major operand, so the
// int8 weights need no unpacking, transposing or register work at all; B = the token
// tile [NT][128 k] (K-major, 128-byte swizzle); D = int32 in TMEM.
//
// Work split (stream-K), as in the W4A16 decode kernel: units are (128-column slab,
// 128-k block); the persistent grid divides them into equal contiguous ranges; a piece
// that covers a whole slab finishes Y itself.  Of a split slab, the piece holding the
// slab's first unit (always its CTA's last piece) finishes it: it waits (bounded) for the
// 64-bit tokens under which the slab's other pieces (always their CTAs' first pieces)
// published their int32 tiles in the workspace, adds them (integer sums, exact in any
// order) and writes Y.  One launch per call.
//
// Roles (256 threads): warp 0 issues TMA; warps 1-2 issue the MMAs, warp 1 + e taking
// the CTA's units i = e (mod 2) (a thread's tcgen05.mma instructions are accepted one
// after another, so two threads keep the tensor core ahead of the weight stream), each
// into its own TMEM accumulators (two per issuer, alternating between slab pieces);
// warps 4-7 run the epilogue (thread = column).  The stage ring has an even depth, so a
// stage always serves the same issuer: every mbarrier has one consumer that waits on
// its phases in order.
#pragma once
#include "common.cuh"

namespace qg {

struct I8DecodeParams {
    const float* t;     // fp32 [M]
    const float* sw;    // fp32 [N]
    uint16_t* Y;        // bf16 [M][N]
    int32_t* dbg;       // NULL or int32 [M][N]: receives acc
    int32_t* partials;  // [grid][NT][128]: the CTA's published piece
    unsigned long long* flags;  // [grid] publication tokens
    unsigned long long token;   // this launch's token (never 0)
    int M, K, N;
    int KB, nslabs, units, grid;  // KB = K / 128 units per slab
};

template <int NT>
struct I8DecCfg {
    static constexpr int W_BYTES = 128 * 128;  // 128 k rows x 128 columns
    static constexpr int X_BYTES = NT * 128;   // NT tokens x 128 k
    static constexpr int STAGE = (W_BYTES + X_BYTES + 1023) / 1024 * 1024;
    static constexpr int ST = NT == 128 ? 6 : 8;  // even: stage s always feeds issuer s % 2
    static_assert(ST % 2 == 0, "stage ring depth must be even");
    static constexpr int EARLY = 4;               // stages whose weights are requested before the wait
    static constexpr int NI = 2, DP = 2;          // issuers, D buffers per issuer
    static constexpr int TMEM_NEED = NI * DP * NT;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                                                      : TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "tensor memory budget");
    static constexpr int THREADS = 256;
    static constexpr int BAR_OFF = ST * STAGE;
    // full[ST] empty[ST] dfull[NI][DP] dempty[NI][DP] done[NI]
    static constexpr int NBAR = 2 * ST + 2 * NI * DP + NI;
    static constexpr int TOTAL = BAR_OFF + NBAR * 8 + 16 + 1024;
};

// idesc: int32 accumulate, A and B signed int8, A MN-major (bit 15), B K-major; N >> 3, M >> 4
__host__ __device__ constexpr uint32_t idesc_s8_amn(int nt)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(nt >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

QG_DEV_INLINE int i8_first_unit(int c, int units, int grid) { return (int)((int64_t)c * units / grid); }

QG_DEV_INLINE int i8_cta_of_unit(int u, int units, int grid)
{
    int c = (int)((int64_t)u * grid / units);
    while (c > 0 && i8_first_unit(c, units, grid) > u) --c;
    while (i8_first_unit(c + 1, units, grid) <= u) ++c;
    return c;
}

// Y (and the debug accumulators) for token t, column n, from the exact sum
QG_DEV_INLINE void i8_finish(const I8DecodeParams& p, int t, int n, int32_t acc, float swn)
{
    const float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), __ldg(p.t + t)), swn);
    p.Y[(int64_t)t * p.N + n] = f32_to_bf16_bits(y);
    if (p.dbg) p.dbg[(int64_t)t * p.N + n] = acc;
}

template <int NT>
__global__ void __launch_bounds__(I8DecCfg<NT>::THREADS, 1)
    w8a8_decode_kernel(const I8DecodeParams p, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_x)
{
    using C = I8DecCfg<NT>;
    constexpr int ST = C::ST, DP = C::DP;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + ST;
    uint64_t* dfull = empty + ST;            // [NI][DP]
    uint64_t* dempty = dfull + C::NI * DP;   // [NI][DP]
    uint64_t* done = dempty + C::NI * DP;    // [NI]
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + C::NI);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = p.KB;
    const int u0 = i8_first_unit(blockIdx.x, p.units, p.grid), u1 = i8_first_unit(blockIdx.x + 1, p.units, p.grid);
    const int n_it = u1 - u0;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < C::NI * DP; ++i) {
            mbar_init(&dfull[i], 1);
            mbar_init(&dempty[i], 128);
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
            // weights do not depend on the previous grid: the first EARLY stages of them
            // are requested before waiting for it; the token tiles after
            int i = 0;
            bool waited = false;
            for (; i < n_it; ++i) {
                const int u = u0 + i, s = i % ST;
                if (!mbar_wait(&empty[s], ((i / ST) & 1) ^ 1)) break;
                uint8_t* st = smem + s * C::STAGE;
                const int slab = u / KB, kb = u % KB;
                mbar_arrive_expect_tx(&full[s], C::W_BYTES + C::X_BYTES);
                tma_load_2d(&tm_w, &full[s], st, slab * 128, kb * 128);
                if (waited) {
                    tma_load_2d(&tm_x, &full[s], st + C::W_BYTES, kb * 128, 0);
                } else if (i + 1 == C::EARLY || i + 1 == n_it) {
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    waited = true;
                    for (int j = 0; j <= i; ++j)
                        tma_load_2d(&tm_x, &full[j % ST], smem + (j % ST) * C::STAGE + C::W_BYTES,
                                    ((u0 + j) % KB) * 128, 0);
                }
            }
            if (!waited) {  // gave up inside the first stages: complete them so that they can land
                asm volatile("griddepcontrol.wait;" ::: "memory");
                for (int j = 0; j < i; ++j)
                    tma_load_2d(&tm_x, &full[j % ST], smem + (j % ST) * C::STAGE + C::W_BYTES, ((u0 + j) % KB) * 128, 0);
            }
            for (int j = i - ST > 0 ? i - ST : 0; j < i; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        }
    } else if (warp <= C::NI) {
        // ---------------- MMA issuers: units i = e (mod 2) ----------------
        if (lane == 0) {
            const int e = warp - 1;
            constexpr uint32_t idesc = idesc_s8_amn(NT);
            bool ok = true, issued = false;
            int i = 0, pc = 0;
            while (ok && i < n_it) {
                // one slab piece: iterations [i, ie)
                const int slab = (u0 + i) / KB;
                const int ie = min(n_it, (slab + 1) * KB - u0);
                const int pb = pc & 1;
                const int d = e * DP + pb;
                if (!mbar_wait(&dempty[d], ((pc >> 1) & 1) ^ 1)) break;  // the epilogue has drained D
                bool first = true;
                for (int it = i + ((e - i) & 1); it < ie; it += 2) {
                    const int s = it % ST;
                    if (!mbar_wait(&full[s], (it / ST) & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t ws = smem_u32(smem + s * C::STAGE);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_i8_ss(tmem + d * NT, smem_desc(ws + 4096 * kk, 16384, 1024, 2),
                                  smem_desc(ws + C::W_BYTES + 32 * kk, 16, 1024, 2), idesc,
                                  (first && kk == 0) ? 0u : 1u);
                    mma_commit(&empty[s]);
                    first = false;
                    issued = true;
                }
                if (!ok) break;
                if (first) mbar_arrive(&dfull[d]);  // no unit of this piece: D holds nothing
                else mma_commit(&dfull[d]);
                i = ie;
                ++pc;
            }
            if (issued) {  // every MMA has completed before tensor memory is released
                mma_commit(&done[e]);
                mbar_wait(&done[e], 0);
            }
        }
    } else if (warp >= 4) {
        // ---------------- epilogue: one thread per column ----------------
        asm volatile("griddepcontrol.wait;" ::: "memory");  // t, sw, Y and the workspace follow the previous grid
        const int q = warp & 3, col = 32 * q + lane;
        const int M = p.M;
        int i = 0, pc = 0;
        bool ok = true;  // after a wait gives up, the schedule is still walked (named barriers) without work
        while (i < n_it) {
            const int slab = (u0 + i) / KB;
            const int ie = min(n_it, (slab + 1) * KB - u0);
            const int pb = pc & 1;
            for (int e = 0; e < C::NI; ++e)
                if (ok && !mbar_wait_backoff(&dfull[e * DP + pb], (pc >> 1) & 1)) ok = false;
            // issuer e holds units of this piece iff some it in [i, ie) has it % 2 == e
            const bool has1 = ie - i >= 2 || ((i & 1) == 1);
            const bool has0 = ie - i >= 2 || ((i & 1) == 0);
            const int n0 = slab * 128, n = n0 + col;
            const bool whole = (u0 + i) % KB == 0 && ie - i == KB;
            const bool head = (u0 + i) % KB == 0 && !whole;  // finishes a split slab (the CTA's last piece)
            int cl = 0;
            if (head) {
                // the slab's other pieces: CTAs blockIdx.x + 1 .. cl
                cl = i8_cta_of_unit(slab * KB + KB - 1, p.units, p.grid);
                bool ready = true;
                if (warp == 4 && ok) ready = watch_tokens(p.flags, (int)blockIdx.x + 1, cl, p.token, lane);
                if (!named_bar_and(1, 128, ok && ready)) ok = false;
            }
            if (ok) {
                tc_fence_after();
                const float swn = ((whole || head) && n < p.N) ? __ldg(p.sw + n) : 0.0f;
                int32_t* mine = p.partials + (size_t)blockIdx.x * NT * 128 + col;
#pragma unroll 1
                for (int t0 = 0; t0 < NT && t0 < M; t0 += 16) {
                    uint32_t a[16], b[16];
                    const uint32_t lanes = (uint32_t)(32 * q) << 16;
                    if (has0) tmem_ld_32x32b_x16(tmem + lanes + (0 * DP + pb) * NT + t0, a);
                    if (has1) tmem_ld_32x32b_x16(tmem + lanes + (1 * DP + pb) * NT + t0, b);
                    tmem_ld_wait();
                    int32_t v[16];
#pragma unroll
                    for (int t = 0; t < 16; ++t) v[t] = (has0 ? (int32_t)a[t] : 0) + (has1 ? (int32_t)b[t] : 0);
                    if (head) {
                        // the other pieces' rows t0 .. t0+15 (inside the NT-row slot even past
                        // M), sixteen loads in flight per piece
                        for (int c = (int)blockIdx.x + 1; c <= cl; ++c) {
                            const int32_t* o = p.partials + (size_t)c * NT * 128 + t0 * 128 + col;
                            int32_t w[16];
#pragma unroll
                            for (int t = 0; t < 16; ++t) w[t] = __ldcg(o + t * 128);
#pragma unroll
                            for (int t = 0; t < 16; ++t) v[t] += w[t];
                        }
                    }
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        if (t0 + t < M) {
                            if (whole || head) {
                                if (n < p.N) i8_finish(p, t0 + t, n, v[t], swn);
                            } else {
                                __stcg(mine + (t0 + t) * 128, v[t]);
                            }
                        }
                    }
                }
                tc_fence_before();
                for (int e = 0; e < C::NI; ++e) mbar_arrive(&dempty[e * DP + pb]);
            }
            if (!whole && !head) {
                // publish: every epilogue thread's stores, then one fence and the token
                named_bar_sync(1, 128);
                if (ok && threadIdx.x == 128) {
                    __threadfence();
                    st_release_u64(p.flags + blockIdx.x, p.token);
                }
            }
            i = ie;
            ++pc;
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
