// tc_gemm.cuh -- tcgen05 tile kernels for prefill-size M (tensor memory accumulators,
// TMA-fed operands, warp-specialised, persistent).
//
// One template covers the two int8 products (KIND); the W4A16 tile kernel, which keeps
// its dequantized weights in tensor memory, is in w4a16_tile.cuh.
//   W8A8  acc = Xq Wq (int8 x int8 -> int32 in TMEM), Y = bf16((acc * t[m]) * sw[n])
//         ("AI Infra guide, ch.4 Quantization" sec. 2.2-2.3, SmoothQuant)
//   W4A8  P_g = Xq q4 per group of 128 (int32 in TMEM, ping-pong), Y = bf16(t[m] sum_g P_g s[g][n])
//         ("LLM inference cost: W8A8/W4A8 ..." sec. 2.2)
//
// Roles (one CTA per SM, persistent over output tiles, n-tile-major order so that
// concurrently running CTAs share the weight tile through L2):
//   warp 0        TMA producer: activation tile and (W8A8) weight tile, or the packed
//                 weight words (W4A8), into a ring of shared-memory stages.
//   warp 1        TMEM allocator and MMA issuer (one elected lane issues tcgen05.mma
//                 and tcgen05.commit; commits release ring stages and publish results).
//   warps 4..     EPI epilogue warps: tcgen05.ld from TMEM, scale, convert, store; epilogue
//                 warp e reads TMEM lanes 32(e%4)..+31 and the e/4-th share of the columns.
//   then          DQ dequant warps (W4A8): unpack nibbles from the raw stage and write
//                 the K-major, 128-byte-swizzled B tile the MMA reads; dequant thread d fills
//                 B row d%128 and the (d/128)-th share of the k-block's words.
// Waits on mbarriers are done by one lane per warp, then __syncwarp.
// Every wait is bounded (mbar_wait); a wait that gives up records QG_ERR_TIMEOUT and
// its role stops issuing work.  No TMA multicast is used anywhere.
#pragma once
#include <climits>

#include "../../include/qgemm.h"
#include "common.cuh"

namespace qg {

// Smallest M routed to the tensor-memory tile kernels (smaller M uses the skinny paths).
constexpr int kTcMinM = 128;
// W4A8 below 128 tokens stays on the skinny kernel (measured faster at 64 tokens).
constexpr int kTcMinMW4A8 = 128;

enum TcKind { TC_W8A8 = 0, TC_W4A8 = 2 };

struct TcW4A16Args {
    const uint16_t* X;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint8_t* zeros;
    uint16_t* Y;
    int M, K, N;
};

struct TcInt8Args {
    const int8_t* Xq;
    const float* t;
    const int8_t* Wq;
    const float* sw;
    const uint32_t* packed;
    const float* sg;
    uint16_t* Y;
    int32_t* dbg;
    int M, K, N;
};

template <int KIND>
struct TcCfg;

// W8A8: tile 128 x 256, k-block 128 int8; A 16 KB + B 32 KB per stage.
template <>
struct TcCfg<TC_W8A8> {
    static constexpr int BM = 128, BN = 256, BK = 128;
    static constexpr int A_BYTES = 128 * 128, B_BYTES = 256 * 128, RAW_BYTES = 0;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int ST = 4;
    static constexpr int EPI = 8, DQ = 0;  // epilogue / dequant warps
    static constexpr int THREADS = 32 * (4 + EPI + DQ);
    static constexpr int TMEM_COLS = 512;  // two 256-column accumulators
};

// W4A8: tile 128 x 128, k-block = one group of 128 int8; A 16 KB, raw 16 x 128 x 4 B = 8 KB,
// B 128 x 128 int8 = 16 KB per stage; TMEM holds two group accumulators (ping-pong); each
// of the 8 epilogue warps keeps the running fp32 sum of its 64 columns in registers.
template <>
struct TcCfg<TC_W4A8> {
    static constexpr int BM = 128, BN = 128, BK = 128;
    static constexpr int A_BYTES = 128 * 128, RAW_BYTES = 16 * 128 * 4, B_BYTES = 128 * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES + RAW_BYTES;
    static constexpr int ST = 4;
    static constexpr int EPI = 8, DQ = 4;   // 8 epilogue warps: each owns 64 columns of a lane quarter
    static constexpr int THREADS = 32 * (4 + EPI + DQ);
    static constexpr int TMEM_COLS = 256;   // two group buffers (ping-pong) of 128 columns
};

template <int KIND>
struct TcSmem {
    using C = TcCfg<KIND>;
    static constexpr int BAR_OFF = C::ST * C::STAGE;
    static constexpr int EPI_OFF = BAR_OFF + 256;         // W4A8: per-epilogue-warp group scales [4][2][128] fp32
    static constexpr int TOTAL = EPI_OFF + (KIND == TC_W4A8 ? C::EPI * 2 * 128 * 4 : 0) + 1024;
};

struct TcParams {
    const float* t;     // W8A8, W4A8: per-token scale
    const float* sw;    // W8A8: per-channel scale
    const float* sg;    // W4A8: per-group scale [K/128][N]
    uint16_t* Y;
    int32_t* dbg;
    int M, K, N;
    int m_tiles, n_tiles;
};

// instruction descriptors (tcgen05 "kind::f16" / "kind::i8"), M = 128
__host__ __device__ constexpr uint32_t idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_s8(int n, bool b_mn_major)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

// bf16x2 of (128 + nibble j, 128 + nibble j+4) -> natural pairs after one subtract and
// one multiply; see the decode kernel for the exponent trick.
QG_DEV_INLINE uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
QG_DEV_INLINE uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// one lane waits, the warp follows; returns the wait's result to every lane
QG_DEV_INLINE bool warp_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_backoff(bar, parity) ? 1u : 0u;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int KIND>
__global__ void __launch_bounds__(TcCfg<KIND>::THREADS, 1)
    tc_gemm_kernel(const TcParams p, const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b)
{
    using C = TcCfg<KIND>;
    using S = TcSmem<KIND>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
    uint64_t* empty = full + C::ST;
    uint64_t* bready = empty + C::ST;      // dequant -> MMA
    uint64_t* tfull = bready + C::ST;      // MMA -> epilogue (2)
    uint64_t* tempty = tfull + 2;          // epilogue -> MMA (2)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = p.K / C::BK;
    const int num_tiles = p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            mbar_init(&bready[i], C::DQ > 0 ? C::DQ : 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], C::EPI);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            int s = 0;
            uint32_t ph = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
                const int m0 = (tile % p.m_tiles) * C::BM, n0 = (tile / p.m_tiles) * C::BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1)) goto producer_done;
                    uint8_t* st = smem + s * C::STAGE;
                    if constexpr (KIND == TC_W8A8) {
                        mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::B_BYTES);
                        tma_load_2d(&tm_a, &full[s], st, kb * 128, m0);
                        tma_load_2d(&tm_b, &full[s], st + C::A_BYTES, n0, kb * 128);
                        tma_load_2d(&tm_b, &full[s], st + C::A_BYTES + 16384, n0 + 128, kb * 128);
                    } else {
                        mbar_arrive_expect_tx(&full[s], C::A_BYTES + C::RAW_BYTES);
                        tma_load_2d(&tm_a, &full[s], st, kb * 128, m0);
                        tma_load_2d(&tm_b, &full[s], st + C::A_BYTES + C::B_BYTES, n0, kb * 16);
                    }
                    if (++s == C::ST) { s = 0; ph ^= 1; }
                }
            }
        }
    producer_done:;
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int li = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++li) {
                if constexpr (KIND == TC_W4A8) {
                    // one TMEM buffer per group, alternating across all groups of all tiles
                    for (int kb = 0; kb < KB; ++kb) {
                        const int gi = li * KB + kb;
                        const int buf = gi & 1;
                        if (!mbar_wait(&tempty[buf], ((gi >> 1) & 1) ^ 1)) { ok = false; break; }
                        if (!mbar_wait(&bready[s], ph)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(smem + s * C::STAGE);
                        const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8_ss(tmem + buf * 128, smem_desc(a0 + 32 * kk, 16, 1024, 2),
                                      smem_desc(b0 + 32 * kk, 16, 1024, 2), idesc_s8(128, false), kk > 0 ? 1u : 0u);
                        mma_commit(&empty[s]);
                        mma_commit(&tfull[buf]);
                        if (++s == C::ST) { s = 0; ph ^= 1; }
                    }
                } else {
                    const int buf = li & 1;
                    if (!mbar_wait(&tempty[buf], ((li >> 1) & 1) ^ 1)) break;
                    tc_fence_after();
                    for (int kb = 0; kb < KB; ++kb) {  // W8A8
                        if (!mbar_wait(&full[s], ph)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a0 = smem_u32(smem + s * C::STAGE);
                        const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_i8_ss(tmem + buf * 256, smem_desc(a0 + 32 * kk, 16, 1024, 2),
                                      smem_desc(b0 + 4096 * kk, 16384, 1024, 2), idesc_s8(256, true), (kb | kk) ? 1u : 0u);
                        mma_commit(&empty[s]);
                        if (++s == C::ST) { s = 0; ph ^= 1; }
                    }
                    if (ok) mma_commit(&tfull[buf]);
                }
            }
        }
    } else if (warp < 4) {
        // warps 2, 3: no role
    } else if (warp < 4 + C::EPI) {
        // ------------------------------ epilogue ------------------------------
        const int e = warp - 4;
        const int q = e & 3;  // TMEM lane quarter this warp may access
        constexpr int CSPLIT = C::EPI / 4;               // warps sharing one lane quarter
        const int cs = e >> 2;                           // this warp's share of the columns
        int li = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
            const int m0 = (tile % p.m_tiles) * C::BM, n0 = (tile / p.m_tiles) * C::BN;
            if constexpr (KIND == TC_W4A8) {
                // Per group: drain the int32 partial P of this warp's CW columns from its TMEM
                // buffer and fold it into the running fp32 sum held in registers:
                //     sum += P * s_g        (exact int32 -> fp32, one fma)
                // Group scales travel global -> register (two groups ahead) -> smem slot (one
                // group ahead) -> broadcast reads, so no load latency sits on the group loop.
                // After the last group the sum is scaled by t[m] and stored as bf16.
                constexpr int CW = C::BN / CSPLIT;   // columns of this warp
                float* sgs = reinterpret_cast<float*>(smem + S::EPI_OFF) + e * 256;
                const int cb = cs * CW;
                const int m = m0 + 32 * q + lane;
                const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16);
                auto load_scales = [&](int g) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    const int n = n0 + cb + 4 * lane;
                    if (4 * lane < CW && g < KB && n < p.N) v = __ldg(reinterpret_cast<const float4*>(p.sg + (int64_t)g * p.N + n));
                    return v;
                };
                auto store_scales = [&](const float4& v, int slot) {
                    if (4 * lane < CW) *reinterpret_cast<float4*>(sgs + slot * 128 + 4 * lane) = v;
                };
                float sum[CW];
#pragma unroll
                for (int i = 0; i < CW; ++i) sum[i] = 0.0f;
                store_scales(load_scales(0), 0);
                float4 s_ahead = load_scales(1);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    const int gi = li * KB + kb;
                    const int buf = gi & 1;
                    store_scales(s_ahead, (kb + 1) & 1);  // group kb+1, loaded one group ago
                    s_ahead = load_scales(kb + 2);
                    __syncwarp();
                    if (!warp_wait(&tfull[buf], (gi >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    const float* sv = sgs + (kb & 1) * 128;
#pragma unroll
                    for (int cc = 0; cc < CW / 32; ++cc) {
                        const int c = cb / 32 + cc;
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(trow + buf * 128 + 32 * c, r);
                        tmem_ld_wait();
                        if (cc == CW / 32 - 1) {       // the whole partial is in registers now
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&tempty[buf]);
                        }
                        if (p.dbg && m < p.M) {
                            int32_t* drow = p.dbg + ((int64_t)m * KB + kb) * p.N + n0 + 32 * c;
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                if (n0 + 32 * c + i < p.N)
                                    *reinterpret_cast<int4*>(drow + i) = make_int4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                        }
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 s4 = *reinterpret_cast<const float4*>(sv + 32 * cc + i);  // broadcast
                            sum[32 * cc + i + 0] = fmaf(i2f_small(r[i + 0]), s4.x, sum[32 * cc + i + 0]);
                            sum[32 * cc + i + 1] = fmaf(i2f_small(r[i + 1]), s4.y, sum[32 * cc + i + 1]);
                            sum[32 * cc + i + 2] = fmaf(i2f_small(r[i + 2]), s4.z, sum[32 * cc + i + 2]);
                            sum[32 * cc + i + 3] = fmaf(i2f_small(r[i + 3]), s4.w, sum[32 * cc + i + 3]);
                        }
                    }
                }
                if (!ok) break;
                if (m < p.M) {
                    const float tm = __ldg(p.t + m);
                    uint16_t* yrow = p.Y + (int64_t)m * p.N + n0 + cb;
#pragma unroll
                    for (int i = 0; i < CW; i += 8) {
                        if (n0 + cb + i < p.N) {
                            uint4 v;
                            v.x = pack_bf16x2_rn(__fmul_rn(tm, sum[i + 0]), __fmul_rn(tm, sum[i + 1]));
                            v.y = pack_bf16x2_rn(__fmul_rn(tm, sum[i + 2]), __fmul_rn(tm, sum[i + 3]));
                            v.z = pack_bf16x2_rn(__fmul_rn(tm, sum[i + 4]), __fmul_rn(tm, sum[i + 5]));
                            v.w = pack_bf16x2_rn(__fmul_rn(tm, sum[i + 6]), __fmul_rn(tm, sum[i + 7]));
                            *reinterpret_cast<uint4*>(yrow + i) = v;
                        }
                    }
                }
            } else {
                const int buf = li & 1;
                if (!warp_wait(&tfull[buf], (li >> 1) & 1)) break;
                tc_fence_after();
                constexpr int NCH = 8 / CSPLIT;  // W8A8: 32-column chunks per warp
                const int m = m0 + 32 * q + lane;
                const float tm = m < p.M ? __ldg(p.t + m) : 0.0f;
#pragma unroll 1
                for (int c = cs * NCH; c < (cs + 1) * NCH; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + buf * 256 + 32 * c, r);
                    tmem_ld_wait();
                    const int nb = n0 + 32 * c;
                    if (m < p.M) {
                        uint16_t* yrow = p.Y + (int64_t)m * p.N + nb;
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            if (nb + i >= p.N) continue;
                            const float4 s0 = __ldg(reinterpret_cast<const float4*>(p.sw + nb + i));
                            const float4 s1 = __ldg(reinterpret_cast<const float4*>(p.sw + nb + i + 4));
                            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(__fmul_rn(__int2float_rn((int)r[i + e]), tm), sv[e]);
                            if (p.dbg) {
                                int32_t* d = p.dbg + (int64_t)m * p.N + nb + i;
                                *reinterpret_cast<int4*>(d) = make_int4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                                *reinterpret_cast<int4*>(d + 4) = make_int4(r[i + 4], r[i + 5], r[i + 6], r[i + 7]);
                            }
                            uint4 v;
                            v.x = pack_bf16x2_rn(f[0], f[1]);
                            v.y = pack_bf16x2_rn(f[2], f[3]);
                            v.z = pack_bf16x2_rn(f[4], f[5]);
                            v.w = pack_bf16x2_rn(f[6], f[7]);
                            *reinterpret_cast<uint4*>(yrow + i) = v;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[buf]);
            }
        }
    } else {
        // ------------------------------ dequant warps (W4A8) ------------------------------
        if constexpr (KIND == TC_W4A8) {
            const int dthr = threadIdx.x - 32 * (4 + C::EPI);
            const int dt = dthr & 127;                 // the B tile row (column n) this thread fills
            constexpr int WSPLIT = C::DQ / 4;           // threads sharing one B row
            const int ws = dthr >> 7;                   // this thread's share of the k-block's words
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!warp_wait(&full[s], ph)) { ok = false; break; }
                    uint8_t* st = smem + s * C::STAGE;
                    const uint32_t* raw = reinterpret_cast<const uint32_t*>(st + C::A_BYTES + C::B_BYTES);
                    uint8_t* brow = st + C::A_BYTES + dt * 128;  // row dt of the K-major B tile
                    {
                        // one group of 128 k = 16 words; two words per 16-byte chunk
#pragma unroll
                        for (int ci = 0; ci < 8 / WSPLIT; ++ci) {
                            const int c = ws * (8 / WSPLIT) + ci;
                            uint32_t o[4];
#pragma unroll
                            for (int hw = 0; hw < 2; ++hw) {
                                const uint32_t word = raw[(2 * c + hw) * 128 + dt];
                                uint32_t ev, od;
                                asm("lop3.b32 %0, %1, 0x0F0F0F0F, 0x08080808, 0x6A;" : "=r"(ev) : "r"(word));
                                asm("lop3.b32 %0, %1, 0x0F0F0F0F, 0x08080808, 0x6A;" : "=r"(od) : "r"(word >> 4));
                                ev = (ev + 0x78787878u) ^ 0x80808080u;
                                od = (od + 0x78787878u) ^ 0x80808080u;
                                o[2 * hw] = prmt(ev, od, 0x5140);
                                o[2 * hw + 1] = prmt(ev, od, 0x7362);
                            }
                            *reinterpret_cast<uint4*>(brow + ((c ^ (dt & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                    fence_proxy_async_smem();  // generic-proxy stores -> visible to tcgen05.mma
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bready[s]);
                    if (++s == C::ST) { s = 0; ph ^= 1; }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing arrives
// at.  mbar_wait gives up after the configured limit and records QG_ERR_TIMEOUT.
__global__ void selftest_wait_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0);
    __syncwarp();
}

}  // namespace qg
