// w4a16_decode.cuh -- decode-shape W4A16 fused dequant-GEMM (M <= 32 per launch).
//
//   Y[m][n] = sum_k X[m][k] (q[k][n] - z[g][n]) s[g][n],   g = k / 128
// ("AI Infra guide, ch.4 Quantization" sec. 3.1 weight-only INT4, sec. 3.5 fused
// INT4 x FP16 kernel; group-wise scale and zero: "LLM inference cost: W8A8/W4A8 ..."
// sec. 2.2).  Decode is a weight stream (0.5 byte per weight): the design keeps HBM
// busy across consecutive calls and the ALU cost per weight small.
//
// Work split (stream-K).  The N columns form slabs of 128; one unit is one group
// (128 k) of one slab.  The grid (at most one CTA per SM) divides the nslabs x G
// units into equal contiguous ranges.  A CTA's range is a list of slab pieces: a piece
// that covers a whole slab writes Y; the piece that holds a split slab's first group
// (always its CTA's last piece) finishes that slab; any other piece of a split slab
// (always its CTA's first piece) publishes its fp32 partial tile in the workspace
// under a per-launch 64-bit token.  The finishing CTA waits (bounded) for the tokens
// of the other pieces, adds their tiles in CTA order (deterministic, no float atomics),
// writes Y and clears the tokens.  One launch per call: no fix-up kernel.
//
// Overlap.  The kernel allows its dependents to launch at once (programmatic dependent
// launch); a CTA of the next call starts on an SM as soon as this call's CTA there exits
// and requests its first ring-full of weights, scales and zeros without waiting for the
// previous grid.  X, Y and the workspace are touched only after griddepcontrol.wait: one
// warp of the producer warpgroup waits and then requests each stage's activations right
// after the stage's weights.
//
// Data movement.  Two producer threads stream into a ring of stages, by TMA: the packed
// words (one 4-D box per stage, [group][32-column block][16 rows][128 B], 128-byte
// swizzled), the fp16 scales and u8 zeros ([group][128 columns]) and the activation
// tile ([half of 64 k][token][128 B], swizzled).  Consumer warp (wn, wg, ws) takes the 64 columns of half wn of group
// wg of every stage, and the ws-th share of its four 32-k steps (one, two or four
// warps per group): more warps hide more latency, fewer steps per warp cost more
// per-group work (scale, zero point, epilogue) per weight.
//
// Math.  Swap-AB mma.sync m16n8k16 (weights are the m16 operand, tokens the n8
// tiles).  A lane's 128-bit read gives 4 columns x 8 k; each nibble pair of a word
// becomes a bf16 (fp16) pair 128 + q (1024 + q) exactly with one shift and one LOP3
// (a multiply-high in place of the shift, to use the FMA pipe, measured slower).  Inside a
// 32-k step the k order is permuted so that a lane's own word feeds its fragment
// slots; the activation pairs get the same permutation with byte permutes.
//   CORR (few tokens): the MMA accumulates D = sum (128 + q) x per group and the zero
//     point and scale are applied once per group and output:
//         acc += s (D - (128 + z) sum x),  sum x from one MMA against an all-ones tile.
//   FULL (more tokens, fewer registers): each pair is dequantized to ((128+q) -
//     (128+z)) * s in the activation dtype (exact subtraction, one rounding), so the
//     MMA accumulates Y directly.
#pragma once
#include "common.cuh"
#include "w4a16_skinny.cuh"

namespace qg {

struct DecodeParams {
    const uint16_t* X;
    const uint16_t* scales;        // fp16 [G][N]
    const uint8_t* zeros;          // u8 [G][N]
    uint16_t* Y;
    float* partials;               // [grid][128 x MP fp32 fragments]
    unsigned long long* flags;     // [grid]
    unsigned long long token;      // this launch's publication token (never 0)
    int M, K, N;
    int G, nslabs, units, grid;
    int narrow;                    // N % 32 != 0: packed words by 2-D boxes per 32-column block
    int ocount;                    // outliers per group and column (the fused side path), 1..4
    uint32_t side_tx;              // side-path bytes of one stage: GPS (2 ocount 128 + 512)
};

constexpr int kDecBN = 128;          // columns per slab
constexpr int kDecGroupW = 8192;     // packed words of one group: 16 rows x 128 columns x 4 B
constexpr int kDecGroupV24 = 4096;   // 2:4 kept codes of one group: 8 rows x 128 columns x 4 B
constexpr int kDecGroupM24 = 2048;   // 2:4 position words of one group: 4 rows x 128 columns x 4 B
constexpr int kDecOutMax = 4;        // outliers per group and column that the fused side path takes

QG_DEV_INLINE int dec_first_unit(int c, int units, int grid) { return (int)((int64_t)c * units / grid); }

// CTA holding unit u of the static split
QG_DEV_INLINE int dec_cta_of_unit(int u, int units, int grid)
{
    int c = (int)((int64_t)u * grid / units);
    while (c > 0 && dec_first_unit(c, units, grid) > u) --c;
    while (dec_first_unit(c + 1, units, grid) <= u) ++c;
    return c;
}

// Shared memory of one CTA: ST stages of GPS groups, the k-warp reduction tiles and
// the stage mbarriers.
template <int MT, int NW, int GPS, int ST, bool PWG, bool SP = false, bool OUT = false>
struct DecodeSmem {
    static constexpr int MP = 8 * MT;
    // weight bytes of one group: packed words, or (2:4) kept codes then position words
    static constexpr int WB = SP ? kDecGroupV24 + kDecGroupM24 : kDecGroupW;
    static constexpr int KW = NW / 2;                 // k-warps per column half
    static constexpr int XG = MP * 256;               // X bytes per group: [2 halves][MP][128 B]
    static constexpr int X_OFF = GPS * WB;
    static constexpr int S_OFF = X_OFF + GPS * XG;    // fp16 scales [GPS][128]
    static constexpr int Z_OFF = S_OFF + GPS * 256;   // u8 zeros [GPS][128]
    // outlier side path (OUT): offsets u8 [GPS][ocount][128], codes i8 [GPS][ocount][128],
    // scales fp32 [GPS][128]
    static constexpr int OI_OFF = Z_OFF + GPS * 128;
    static constexpr int OC_OFF = OI_OFF + GPS * kDecOutMax * 128;
    static constexpr int OS_OFF = OC_OFF + GPS * kDecOutMax * 128;
    static constexpr int END = OUT ? OS_OFF + GPS * 512 : Z_OFF + GPS * 128;
    static constexpr int STAGE = (END + 1023) / 1024 * 1024;
    static constexpr int FRAG = 4 * MT;               // float4 accumulator fragments per lane (64 columns x MP tokens per warp)
    static constexpr int TS = kDecBN + 4;            // row stride (floats) of the [token][column] result tile
    static constexpr int RED_K = (KW - 1) * 2 * FRAG * 32 * 16;  // k-warp reduction (fragment layout)
    static constexpr int RED = RED_K > MP * TS * 4 ? RED_K : MP * TS * 4;  // the result tile aliases it
    static constexpr int SIDE = OUT ? 2 * MP * kDecBN * 4 : 0;  // side-path sums of a piece, 2 x [token][128] fp32
    static constexpr int TOTAL = ST * STAGE + RED + SIDE + 3 * ST * 8 + 16 + 1024;
    // The producer is a whole warpgroup after the consumers, whose first two warps issue
    // (the weights, the activations) and, with the side path, whose last two sum it, so
    // that the register file can be split with setmaxnreg: the producer warps keep 56
    // registers a thread (136 with the side path) and the consumers take the rest.  (Two
    // bare issuer warps without the split measured slower.)
    static constexpr int THREADS = 32 * NW + 128;
    static constexpr int REG_LAUNCH = (65536 / THREADS) / 8 * 8 > 255 ? 248 : (65536 / THREADS) / 8 * 8;
    static constexpr int REG_PRODUCER = OUT ? 136 : 56;
    static constexpr int REG_CONSUMER_RAW = (REG_LAUNCH * THREADS - REG_PRODUCER * 128) / (32 * NW) / 8 * 8;
    static constexpr int REG_CONSUMER = REG_CONSUMER_RAW > 248 ? 248 : REG_CONSUMER_RAW;
    static constexpr uint32_t GROUP_TX = WB + XG + 384;  // TMA bytes of one group
    static constexpr int PARTIAL_FLOATS = 2 * FRAG * 32 * 4;  // one CTA's partial tile (128 x MP)
};

// Tensor maps.  Packed words: 4-D {32 columns, 16 rows, N/32 blocks, G groups} with
// boxes of GPS groups or 1 group, landing as [group][block][16 rows][128 B]; when
// N % 32 != 0, 2-D boxes {32 columns, 16 rows} per block and group into the same
// layout.  Activations: 3-D {64 k, M rows, K/64 halves}, boxes of 2 GPS or 2 halves.
struct DecodeMaps {
    CUtensorMap sg, s1, zg, z1;  // fp16 scales / u8 zeros: {128 columns, GPS | 1 groups}
    CUtensorMap wg, w1;  // packed words, GPS groups / 1 group (4-D), or the 2-D per-block map in w1
    CUtensorMap xg, x1;  // activations, GPS groups / 1 group
    CUtensorMap mg, m1;  // 2:4 position words {32 columns, 4 rows, N/32 blocks, G groups}, GPS groups / 1 group
    CUtensorMap oi, oc, os;  // outlier offsets / codes {N, ocount, G} and scales {N, G}, GPS groups
};

QG_DEV_INLINE void tma_load_4d(const CUtensorMap* m, uint64_t* bar, void* smem_dst, int x, int y, int z, int w)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
        "%6}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

// Walks a CTA's schedule: pieces (runs of groups within one slab) in order, each cut
// into stages of at most GPS groups.  Producer and consumers walk the same schedule.
struct DecodeSchedule {
    int u, u1, G;
    int slab, ga, gb;  // current piece
    QG_DEV_INLINE DecodeSchedule(int u0_, int u1_, int G_) : u(u0_), u1(u1_), G(G_) { set_piece(); }
    QG_DEV_INLINE void set_piece()
    {
        slab = u / G;
        ga = u % G;
        gb = min(G, ga + (u1 - u));
    }
    QG_DEV_INLINE bool done() const { return u >= u1; }
    QG_DEV_INLINE void next_piece()
    {
        u += gb - ga;
        if (u < u1) set_piece();
    }
};

template <int MT, bool BF16, int NW, int GPS, int ST, bool FULL, bool PWG, int MINB, bool SP, bool OUT>
__global__ void __launch_bounds__(DecodeSmem<MT, NW, GPS, ST, PWG, SP, OUT>::THREADS, MINB)
    w4a16_decode_kernel(const DecodeParams p, const __grid_constant__ DecodeMaps maps)
{
    using H = HalfOps<BF16>;
    using L = DecodeSmem<MT, NW, GPS, ST, PWG, SP, OUT>;
    static_assert(!(SP && OUT), "the side path is fused into the dense kernel only");
    static_assert(!SP || FULL, "the 2:4 path dequantizes in full");
    constexpr int MP = L::MP;
    constexpr int KW = L::KW;
    constexpr int WS = KW / GPS;   // warps sharing one group of a column half
    constexpr int SPW = 4 / WS;    // 32-k steps per warp and group
    static_assert(KW == GPS * WS && (WS == 1 || WS == 2 || WS == 4), "consumer warps: 2 x groups x step shares");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float4* red = reinterpret_cast<float4*>(smem + ST * L::STAGE);
    float* side = reinterpret_cast<float*>(smem + ST * L::STAGE + L::RED);  // 2 x [MP][128] (OUT)
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * L::STAGE + L::RED + L::SIDE);
    uint64_t* empty = full + ST;
    uint64_t* armed = empty + ST;  // the producer has set up a stage's fill (its expected bytes)
    volatile int* side_fail = reinterpret_cast<volatile int*>(armed + ST);  // a side-path wait gave up (OUT)
    constexpr int NSIDE = OUT ? 2 : 0;  // side-path warps: NW + 2, NW + 3
    constexpr int SIDEBAR = 32 * (NW + NSIDE);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;
    const int u0 = dec_first_unit(blockIdx.x, p.units, p.grid), u1 = dec_first_unit(blockIdx.x + 1, p.units, p.grid);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NW + NSIDE);
            mbar_init(&armed[i], 1);
        }
        *side_fail = 0;
        fence_mbar_init();
    }
    __syncthreads();

    static_assert(PWG, "the producer warpgroup holds the weight and the activation issuers");
    if (warp >= NW) {
        // ---------------- producer warpgroup ----------------
        // Warp NW streams the weights (with scales and zeros) from the start: they do not
        // depend on the previous grid.  Warp NW + 1 waits for the previous grid once and
        // then requests each fill's activations as soon as the weight issuer has set the
        // fill up, so a CTA that starts late (after the previous grid ended) gets its first
        // stage's activations right behind that stage's weights, not behind the whole ring.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(L::REG_PRODUCER));
        if constexpr (OUT) {
            if (warp >= NW + 2) {
                // ---------------- outlier side path (warps NW + 2, NW + 3) ----------------
                // Side warp sw (0, 1) takes the groups gi = sw, sw + 2, .. of every stage; its
                // lane l takes columns 4l .. 4l + 3 (one 4-byte load gives an outlier slot of
                // all four).  Per group: sums[m][c] += sum_r x[m][g 128 + idx_r] (code_r s8),
                // in group then slot order, into the warp's own sums; at the piece's end both
                // warps' sums are in shared memory and the consumers add them to the piece's
                // tile (so Y is rounded once).  The warps walk the same schedule as the
                // consumers and release each stage with them.
                const int sw = warp - (NW + 2), c0 = 4 * lane;
                const int cnt = p.ocount, M = p.M;
                float* mine = side + sw * (MP * kDecBN);
                // up to 8 tokens the piece's sums stay in registers; with more a group's sums
                // are added to the warp's shared-memory sums
                constexpr bool SREG = MP <= 8;
                float sacc[4][SREG ? MP : 1];
                int stage = 0;
                uint32_t phase = 0;
                bool sok = true, bad = false;
                DecodeSchedule sc(u0, u1, G);
                for (bool firstp = true; !sc.done(); sc.next_piece(), firstp = false) {
                    if constexpr (SREG) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
#pragma unroll
                            for (int m = 0; m < MP; ++m) sacc[j][m] = 0.0f;
                    } else {
                        if (!firstp) named_bar_sync(3, SIDEBAR);  // the consumers took the previous piece's sums
                        for (int m = 0; m < MP; ++m)
                            *reinterpret_cast<float4*>(mine + m * kDecBN + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    for (int g0 = sc.ga; g0 < sc.gb; g0 += GPS) {
                        const int ng = min(GPS, sc.gb - g0);
                        if (sok && !mbar_wait_backoff(&full[stage], phase)) sok = false;
                        if (sok) {
                            const uint8_t* st = ring + stage * L::STAGE;
                            // groups one at a time: the side code stays small beside the
                            // consumers' loop in the instruction cache
#pragma unroll 1
                            for (int gg = 0; gg < (GPS + 1) / 2; ++gg) {
                                const int gi = 2 * gg + sw;
                                if (gi < ng) {
                                    // the group's slots for the four columns: offsets, weights
                                    const float4 s4 = *reinterpret_cast<const float4*>(st + L::OS_OFF + (gi * kDecBN + c0) * 4);
                                    const float s8v[4] = {s4.x, s4.y, s4.z, s4.w};
                                    uint32_t i4[kDecOutMax], q4[kDecOutMax];
#pragma unroll
                                    for (int r = 0; r < kDecOutMax; ++r) {
                                        i4[r] = r < cnt ? *reinterpret_cast<const uint32_t*>(st + L::OI_OFF + (gi * cnt + r) * kDecBN + c0) : 0u;
                                        q4[r] = r < cnt ? *reinterpret_cast<const uint32_t*>(st + L::OC_OFF + (gi * cnt + r) * kDecBN + c0) : 0u;
                                    }
                                    const uint8_t* xgrp = st + L::X_OFF + gi * L::XG;
                                    if (M == 1) {
                                        // one token (row 0 of the tile, no swizzle offset): a
                                        // loop of its own, so the code it runs stays compact
#pragma unroll
                                        for (int j = 0; j < 4; ++j) {
                                            float g1 = SREG ? sacc[j][0] : 0.0f;
#pragma unroll
                                            for (int r = 0; r < kDecOutMax; ++r) {
                                                if (r < cnt) {
                                                    const int k = (int)((i4[r] >> (8 * j)) & 0xFFu);
                                                    const float w = __fmul_rn(i2f_small((uint32_t)(int32_t)(int8_t)((q4[r] >> (8 * j)) & 0xFFu)), s8v[j]);
                                                    if (k >= kDecBN) {  // not an offset inside the group: skipped, reported
                                                        bad = true;
                                                        continue;
                                                    }
                                                    const uint16_t xb = *reinterpret_cast<const uint16_t*>(
                                                        xgrp + (k >> 6) * (MP * 128) + (k & 7) * 2 + (((k & 63) >> 3) << 4));
                                                    const float xv = BF16 ? bf16_bits_to_f32(xb) : __half2float(__ushort_as_half(xb));
                                                    g1 = fmaf(xv, w, g1);
                                                }
                                            }
                                            if constexpr (SREG) sacc[j][0] = g1;
                                            else mine[c0 + j] += g1;
                                        }
                                    } else {
                                    // the four columns one at a time when the sums live in shared
                                    // memory (more than 8 tokens): a quarter of the code
#pragma unroll(SREG ? 4 : 1)
                                    for (int j = 0; j < 4; ++j) {
                                        const float sj = (j & 2) ? ((j & 1) ? s4.w : s4.z) : ((j & 1) ? s4.y : s4.x);
                                        float gacc[MP];
#pragma unroll
                                        for (int m = 0; m < MP; ++m) gacc[m] = SREG ? sacc[j][SREG ? m : 0] : 0.0f;
#pragma unroll
                                        for (int r = 0; r < kDecOutMax; ++r) {
                                            if (r < cnt) {
                                                int k = (int)((i4[r] >> (8 * j)) & 0xFFu);
                                                const float w = __fmul_rn(i2f_small((uint32_t)(int32_t)(int8_t)((q4[r] >> (8 * j)) & 0xFFu)), sj);
                                                if (k >= kDecBN) {  // not an offset inside the group: skipped, reported
                                                    bad = true;
                                                    continue;
                                                }
                                                const uint8_t* xk = xgrp + (k >> 6) * (MP * 128) + (k & 7) * 2;
                                                const int ch = (k & 63) >> 3;
#pragma unroll
                                                for (int mb = 0; mb < MP / 8; ++mb) {
                                                    if (8 * mb < M) {
#pragma unroll
                                                        for (int mm = 0; mm < 8; ++mm) {
                                                            const int m = 8 * mb + mm;
                                                            if (m < M) {
                                                                const uint16_t xb = *reinterpret_cast<const uint16_t*>(xk + m * 128 + ((ch ^ (m & 7)) << 4));
                                                                const float xv = BF16 ? bf16_bits_to_f32(xb) : __half2float(__ushort_as_half(xb));
                                                                gacc[m] = fmaf(xv, w, gacc[m]);
                                                            }
                                                        }
                                                    }
                                                }
                                            }
                                        }
                                        if constexpr (SREG) {
#pragma unroll
                                            for (int m = 0; m < MP; ++m) sacc[j][SREG ? m : 0] = gacc[m];
                                        } else {
#pragma unroll
                                            for (int m = 0; m < MP; ++m)
                                                if (m < M) mine[m * kDecBN + c0 + j] += gacc[m];
                                        }
                                    }
                                    }
                                }
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&empty[stage]);
                        if (++stage == ST) { stage = 0; phase ^= 1; }
                    }
                    if constexpr (SREG) {
                        if (!firstp) named_bar_sync(3, SIDEBAR);  // the consumers took the previous piece's sums
#pragma unroll
                        for (int m = 0; m < MP; ++m)
                            *reinterpret_cast<float4*>(mine + m * kDecBN + c0) = make_float4(sacc[0][SREG ? m : 0], sacc[1][SREG ? m : 0],
                                                                                           sacc[2][SREG ? m : 0], sacc[3][SREG ? m : 0]);
                    }
                    if (!sok) *side_fail = 1;
                    named_bar_arrive(2, SIDEBAR);  // this piece's side sums are complete
                }
                if (bad) set_status(6u);
                named_bar_sync(3, SIDEBAR);
                return;
            }
        } else {
            if (warp > NW + 1) return;
        }
        if (warp == NW + 1) {
            if (lane == 0) {
                tma_prefetch_desc(&maps.xg);
                tma_prefetch_desc(&maps.x1);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int stage = 0;
            uint32_t phase = 0;
            DecodeSchedule sc(u0, u1, G);
            for (bool ok = true; !sc.done() && ok; sc.next_piece()) {
                for (int g0 = sc.ga; g0 < sc.gb; g0 += GPS) {
                    const int ng = min(GPS, sc.gb - g0);
                    if (!__all_sync(0xffffffffu, mbar_wait(&armed[stage], phase))) { ok = false; break; }
                    if (lane == 0) {
                        uint8_t* st = ring + stage * L::STAGE;
                        if (ng == GPS)
                            tma_load_3d(&maps.xg, &full[stage], st + L::X_OFF, 0, 0, 2 * g0);
                        else
                            for (int i = 0; i < ng; ++i)
                                tma_load_3d(&maps.x1, &full[stage], st + L::X_OFF + i * L::XG, 0, 0, 2 * (g0 + i));
                    }
                    if (++stage == ST) { stage = 0; phase ^= 1; }
                }
            }
            return;
        }
        if (lane == 0) {
            tma_prefetch_desc(&maps.wg);
            tma_prefetch_desc(&maps.w1);
            if constexpr (OUT) {
                tma_prefetch_desc(&maps.oi);
                tma_prefetch_desc(&maps.oc);
                tma_prefetch_desc(&maps.os);
            }
            if constexpr (SP) {
                tma_prefetch_desc(&maps.mg);
                tma_prefetch_desc(&maps.m1);
            }
        }
        int stage = 0, issued = 0;
        uint32_t phase = 0;
        bool ok = true;
        DecodeSchedule sc(u0, u1, G);
        for (; !sc.done() && ok; sc.next_piece()) {
            const int x = sc.slab * kDecBN;
            for (int g0 = sc.ga; g0 < sc.gb; g0 += GPS) {
                const int ng = min(GPS, sc.gb - g0);
                // every lane waits (acquiring the consumers' release of the stage); a lane that
                // gave up makes the whole warp stop
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1))) { ok = false; break; }
                uint8_t* st = ring + stage * L::STAGE;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)ng * L::GROUP_TX + (OUT ? p.side_tx : 0u));
                    if constexpr (OUT) {
                        // always GPS groups (groups past G read as zero; others unused)
                        tma_load_3d(&maps.oi, &full[stage], st + L::OI_OFF, x, 0, g0);
                        tma_load_3d(&maps.oc, &full[stage], st + L::OC_OFF, x, 0, g0);
                        tma_load_2d(&maps.os, &full[stage], st + L::OS_OFF, x, g0);
                    }
                    if constexpr (SP) {
                        // kept codes [group][block][8 rows][128 B], then position words
                        // [group][block][4 rows][128 B]
                        if (ng == GPS) {
                            tma_load_4d(&maps.wg, &full[stage], st, 0, 0, x / 32, g0);
                            tma_load_4d(&maps.mg, &full[stage], st + GPS * kDecGroupV24, 0, 0, x / 32, g0);
                        } else {
                            for (int i = 0; i < ng; ++i) {
                                tma_load_4d(&maps.w1, &full[stage], st + i * kDecGroupV24, 0, 0, x / 32, g0 + i);
                                tma_load_4d(&maps.m1, &full[stage], st + GPS * kDecGroupV24 + i * kDecGroupM24, 0, 0,
                                            x / 32, g0 + i);
                            }
                        }
                    } else if (p.narrow) {
                        for (int i = 0; i < ng; ++i)
#pragma unroll
                            for (int b = 0; b < 4; ++b)
                                tma_load_2d(&maps.w1, &full[stage], st + i * kDecGroupW + b * 2048, x + 32 * b,
                                            16 * (g0 + i));
                    } else if (ng == GPS) {
                        tma_load_4d(&maps.wg, &full[stage], st, 0, 0, x / 32, g0);
                    } else {
                        for (int i = 0; i < ng; ++i)
                            tma_load_4d(&maps.w1, &full[stage], st + i * kDecGroupW, 0, 0, x / 32, g0 + i);
                    }
                    if (ng == GPS) {
                        tma_load_2d(&maps.sg, &full[stage], st + L::S_OFF, x, g0);
                        tma_load_2d(&maps.zg, &full[stage], st + L::Z_OFF, x, g0);
                    } else {
                        for (int i = 0; i < ng; ++i) {
                            tma_load_2d(&maps.s1, &full[stage], st + L::S_OFF + i * 256, x, g0 + i);
                            tma_load_2d(&maps.z1, &full[stage], st + L::Z_OFF + i * 128, x, g0 + i);
                        }
                    }
                    mbar_arrive(&armed[stage]);  // the activation issuer may now add its copy
                }
                ++issued;
                if (++stage == ST) { stage = 0; phase ^= 1; }
            }
        }
        // every TMA copy still in flight lands before the CTA exits (bounded waits: a fill
        // whose activations were never requested gives up)
        if (lane == 0)
            for (int j = issued - ST > 0 ? issued - ST : 0; j < issued; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        return;
    }

    // ---------------- consumers ----------------
    if constexpr (PWG) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(L::REG_CONSUMER));
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int wn = warp & 1, wk = warp >> 1;
    const int wg = wk / WS, ws = wk % WS;  // this warp's group of a stage and share of its steps
    const int g8 = lane >> 2, t4 = lane & 3;
    const uint32_t ONE = BF16 ? 0x3F803F80u : 0x3C003C00u;
    float acc[2][2][MT][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < MT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[h][c][j][e] = 0.0f;

    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    DecodeSchedule sc(u0, u1, G);
    // After a wait gives up (status recorded) the warp keeps walking the schedule
    // without waiting or computing, so that every named barrier still sees all
    // consumer threads; nothing is written to global memory after that.
    for (; !sc.done(); sc.next_piece()) {
        for (int g0 = sc.ga; g0 < sc.gb; g0 += GPS) {
            const int ng = min(GPS, sc.gb - g0);
            if (ok && !mbar_wait_backoff(&full[stage], phase)) ok = false;
            const uint8_t* st = ring + stage * L::STAGE;
            if (ok && wg < ng) {
                {
                    const int gi = wg;
                    // scale and zero of the lane's 8 columns (4 per 32-column block h): the
                    // full dequantization needs them during the steps, the per-group
                    // correction only at the group's end (fewer live registers)
                    auto col_sz = [&](int h, int c, float& s, float& zb) {
                        const int col = 64 * wn + 32 * h + 4 * g8 + c;
                        s = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(st + L::S_OFF + gi * 256 + col * 2)));
                        zb = H::BIAS + (float)st[L::Z_OFF + gi * 128 + col];
                    };
                    uint32_t s2[2][4], z2[2][4];
                    if constexpr (FULL) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                float sv, zb;
                                col_sz(h, c, sv, zb);
                                s2[h][c] = H::splat(sv);   // bf16: s rounded once; fp16: exact
                                z2[h][c] = H::splat(zb);   // exact (integer <= 143, or 1024 + z)
                            }
                    }
                    if constexpr (SP) {
                        // 2:4: mma.sp m16n8k32, weights compressed (two kept codes of each
                        // 4-block) as the m16 operand.  The lane's kept-code words: rows
                        // 2 t4 (its block t4 of each step) and 2 t4 + 1 (block t4 + 4) of
                        // columns 4 g8 .. 4 g8 + 3; nibble pair s of a word (bits 4s and 16 + 4s)
                        // is step s's pair, extracted with one shift and one LOP3.
                        const uint8_t* vbase = st + gi * kDecGroupV24;
                        const uint8_t* mbase = st + GPS * kDecGroupV24 + gi * kDecGroupM24;
                        const uint8_t* xgrp = st + L::X_OFF + gi * L::XG;
                        uint4 va[2][2];
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int hb = 0; hb < 2; ++hb)
                                va[h][hb] = *reinterpret_cast<const uint4*>(vbase + (2 * wn + h) * 1024 +
                                                                            (2 * t4 + hb) * 128 + g8 * 16);
                        // position words: lanes t4 = 0 / 1 give the MMA blocks 0-3 / 4-7 of
                        // both rows (selector 0); the other lanes' are not read
                        const uint32_t msel = (t4 & 1) ? 0x7632u : 0x5410u;
#pragma unroll
                        for (int si = 0; si < SPW; ++si) {
                            const int s = ws * SPW + si;
                            // activations in natural k order: B rows 2 t4 + 8 i (+1), i = 0..3
                            uint32_t xb[MT][4];
                            const uint8_t* xs = xgrp + (s >> 1) * (MP * 128);
#pragma unroll
                            for (int j = 0; j < MT; ++j) {
                                const int tok = 8 * j + g8;  // rows >= M are zero (TMA fill)
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    xb[j][i] = *reinterpret_cast<const uint32_t*>(
                                        xs + tok * 128 + (((4 * (s & 1) + i) ^ (tok & 7)) << 4) + 4 * t4);
                            }
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                const uint4 mv = *reinterpret_cast<const uint4*>(mbase + (2 * wn + h) * 512 + s * 128 + g8 * 16);
                                const uint32_t w0[4] = {va[h][0].x, va[h][0].y, va[h][0].z, va[h][0].w};
                                const uint32_t w1[4] = {va[h][1].x, va[h][1].y, va[h][1].z, va[h][1].w};
#pragma unroll
                                for (int cp = 0; cp < 2; ++cp) {
                                    // MMA row g8 <-> column 4 g8 + 2 cp, row g8 + 8 <-> column 4 g8 + 2 cp + 1
                                    uint32_t a0 = lop3_and_or(w0[2 * cp] >> (4 * s), 0x000F000Fu, H::MAGIC);
                                    uint32_t a1 = lop3_and_or(w0[2 * cp + 1] >> (4 * s), 0x000F000Fu, H::MAGIC);
                                    uint32_t a2 = lop3_and_or(w1[2 * cp] >> (4 * s), 0x000F000Fu, H::MAGIC);
                                    uint32_t a3 = lop3_and_or(w1[2 * cp + 1] >> (4 * s), 0x000F000Fu, H::MAGIC);
                                    a0 = H::mul2(H::sub2(a0, z2[h][2 * cp]), s2[h][2 * cp]);
                                    a1 = H::mul2(H::sub2(a1, z2[h][2 * cp + 1]), s2[h][2 * cp + 1]);
                                    a2 = H::mul2(H::sub2(a2, z2[h][2 * cp]), s2[h][2 * cp]);
                                    a3 = H::mul2(H::sub2(a3, z2[h][2 * cp + 1]), s2[h][2 * cp + 1]);
                                    const uint32_t meta = prmt(cp ? mv.z : mv.x, cp ? mv.w : mv.y, msel);
#pragma unroll
                                    for (int j = 0; j < MT; ++j)
                                        mma_sp_16832<BF16>(acc[h][cp][j], a0, a1, a2, a3, xb[j][0], xb[j][1], xb[j][2],
                                                           xb[j][3], meta);
                                }
                            }
                        }
                    } else {
                    float D[2][2][MT][4], Dx[MT][4];
                    if constexpr (!FULL) {
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) Dx[j][e] = 0.0f;
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int c = 0; c < 2; ++c)
#pragma unroll
                                    for (int e = 0; e < 4; ++e) D[h][c][j][e] = 0.0f;
                        }
                    }
                    const uint8_t* wbase = st + gi * kDecGroupW;
                    const uint8_t* xgrp = st + L::X_OFF + gi * L::XG;
#pragma unroll
                    for (int si = 0; si < SPW; ++si) {
                        const int s = ws * SPW + si;
                        const int row = 8 * (s >> 1) + 2 * t4 + (s & 1);  // packed-word row within the group
                        uint4 wv[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            wv[h] = *reinterpret_cast<const uint4*>(wbase + (2 * wn + h) * 2048 + row * 128 +
                                                                    ((g8 ^ (row & 7)) << 4));
                        uint32_t xb[MT][4];
                        const uint8_t* xs = xgrp + (row >> 3) * (MP * 128);
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const int tok = 8 * j + g8;  // rows >= M are zero (TMA fill)
                            const uint4 xv =
                                *reinterpret_cast<const uint4*>(xs + tok * 128 + (((row & 7) ^ (tok & 7)) << 4));
                            xb[j][0] = prmt(xv.x, xv.z, 0x5410);
                            xb[j][1] = prmt(xv.x, xv.z, 0x7632);
                            xb[j][2] = prmt(xv.y, xv.w, 0x5410);
                            xb[j][3] = prmt(xv.y, xv.w, 0x7632);
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t w[4] = {wv[h].x, wv[h].y, wv[h].z, wv[h].w};
                            uint32_t R[4][4];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                R[c][0] = lop3_and_or(w[c], 0x000F000Fu, H::MAGIC);
                                R[c][1] = lop3_and_or(w[c] >> 4, 0x000F000Fu, H::MAGIC);
                                R[c][2] = lop3_and_or(w[c] >> 8, 0x000F000Fu, H::MAGIC);
                                R[c][3] = lop3_and_or(w[c] >> 12, 0x000F000Fu, H::MAGIC);
                                if constexpr (FULL) {
#pragma unroll
                                    for (int r = 0; r < 4; ++r) R[c][r] = H::mul2(H::sub2(R[c][r], z2[h][c]), s2[h][c]);
                                }
                            }
#pragma unroll
                            for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                                for (int j = 0; j < MT; ++j) {
                                    if constexpr (FULL) {
                                        mma_16816<BF16>(acc[h][cp][j], R[2 * cp][0], R[2 * cp + 1][0], R[2 * cp][1],
                                                        R[2 * cp + 1][1], xb[j][0], xb[j][1]);
                                        mma_16816<BF16>(acc[h][cp][j], R[2 * cp][2], R[2 * cp + 1][2], R[2 * cp][3],
                                                        R[2 * cp + 1][3], xb[j][2], xb[j][3]);
                                    } else {
                                        mma_16816<BF16>(D[h][cp][j], R[2 * cp][0], R[2 * cp + 1][0], R[2 * cp][1],
                                                        R[2 * cp + 1][1], xb[j][0], xb[j][1]);
                                        mma_16816<BF16>(D[h][cp][j], R[2 * cp][2], R[2 * cp + 1][2], R[2 * cp][3],
                                                        R[2 * cp + 1][3], xb[j][2], xb[j][3]);
                                    }
                                }
                        }
                        if constexpr (!FULL) {
#pragma unroll
                            for (int j = 0; j < MT; ++j) {
                                mma_16816<BF16>(Dx[j], ONE, ONE, ONE, ONE, xb[j][0], xb[j][1]);
                                mma_16816<BF16>(Dx[j], ONE, ONE, ONE, ONE, xb[j][2], xb[j][3]);
                            }
                        }
                    }
                    if constexpr (!FULL) {
                        // group epilogue (this warp's steps): acc += s (D - (128 + z) sum x)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                float sv, zb;
                                col_sz(h, c, sv, zb);
                                const int cp = c >> 1, e0 = 2 * (c & 1);  // fragment elements of column c
#pragma unroll
                                for (int j = 0; j < MT; ++j)
#pragma unroll
                                    for (int e = e0; e < e0 + 2; ++e)
                                        acc[h][cp][j][e] = fmaf(sv, fmaf(-zb, Dx[j][e & 1], D[h][cp][j][e]), acc[h][cp][j][e]);
                            }
                    }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == ST) { stage = 0; phase ^= 1; }
        }

        // ---------------- piece end ----------------
        // 1. the k-warps of each column half add into warp (wn, 0), in wk order
        if constexpr (KW > 1) {
            if (wk > 0) {
                float4* dst = red + ((wk - 1) * 2 + wn) * L::FRAG * 32;
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                        for (int j = 0; j < MT; ++j) {
                            const int i = (h * 2 + cp) * MT + j;
                            dst[i * 32 + lane] = make_float4(acc[h][cp][j][0], acc[h][cp][j][1], acc[h][cp][j][2],
                                                             acc[h][cp][j][3]);
                        }
            }
            named_bar_sync(1, 32 * NW);
            if (wk == 0) {
#pragma unroll 1
                for (int q = 1; q < KW; ++q) {
                    const float4* src = red + ((q - 1) * 2 + wn) * L::FRAG * 32;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                            for (int j = 0; j < MT; ++j) {
                                const float4 v = src[((h * 2 + cp) * MT + j) * 32 + lane];
                                acc[h][cp][j][0] += v.x;
                                acc[h][cp][j][1] += v.y;
                                acc[h][cp][j][2] += v.z;
                                acc[h][cp][j][3] += v.w;
                            }
                }
            }
        }
        // any consumer warp that gave up makes the whole CTA skip its global writes
        const int all_ok = named_bar_and(1, 32 * NW, ok);
        if (!all_ok) ok = false;

        // 2. warps (0, 0) and (1, 0) hold the piece's 128 x MP result: into the tile
        //    [token][column] (row stride TS floats), which aliases the reduction area
        float* tile = reinterpret_cast<float*>(red);
        if (wk == 0 && ok) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const int col = 64 * wn + 32 * h + 4 * g8 + 2 * cp, tok = 8 * j + 2 * t4;
                        *reinterpret_cast<float2*>(tile + tok * L::TS + col) = make_float2(acc[h][cp][j][0], acc[h][cp][j][2]);
                        *reinterpret_cast<float2*>(tile + (tok + 1) * L::TS + col) =
                            make_float2(acc[h][cp][j][1], acc[h][cp][j][3]);
                    }
        }
        named_bar_sync(1, 32 * NW);
        if constexpr (OUT) {
            // the side-path warps' sums of this piece: add them to the tile (each thread the
            // elements it takes in step 3); the side warps overwrite them for the next piece
            // only after the arrival below
            named_bar_sync(2, SIDEBAR);
            if (*side_fail) ok = false;
            for (int e = threadIdx.x; e < MP * 32; e += 32 * NW) {
                float4* tv = reinterpret_cast<float4*>(tile + (e >> 5) * L::TS + 4 * (e & 31));
                const float4 a = *tv, b = *reinterpret_cast<const float4*>(side + (e >> 5) * kDecBN + 4 * (e & 31)),
                             c = *reinterpret_cast<const float4*>(side + MP * kDecBN + (e >> 5) * kDecBN + 4 * (e & 31));
                *tv = make_float4(a.x + (b.x + c.x), a.y + (b.y + c.y), a.z + (b.z + c.z), a.w + (b.w + c.w));
            }
            named_bar_arrive(3, SIDEBAR);
        }

        // 3. every consumer thread takes float4 elements (token, 4 columns) of the tile
        if (ok) {
            constexpr int NE = MP * 32;             // float4 elements of the tile
            constexpr int EPT = (NE + 32 * NW - 1) / (32 * NW);
            const int ct = threadIdx.x;             // 0 .. 32 NW - 1
            const bool whole = sc.ga == 0 && sc.gb == G;
            const bool head = sc.ga == 0 && !whole;  // finishes a split slab (the CTA's last piece)
            const int n0 = sc.slab * kDecBN;
            if (!whole && !head) {
                // publish this piece's tile ([token][128 columns] fp32), then its token: the
                // barrier orders every thread's stores before the one fence and release
                float4* mine = reinterpret_cast<float4*>(p.partials) + (size_t)blockIdx.x * (L::PARTIAL_FLOATS / 4);
#pragma unroll
                for (int i = 0; i < EPT; ++i) {
                    const int e = ct + i * 32 * NW;
                    if (e < NE) __stcg(mine + e, *reinterpret_cast<const float4*>(tile + (e >> 5) * L::TS + 4 * (e & 31)));
                }
                named_bar_sync(1, 32 * NW);
                if (ct == 0) {
                    __threadfence();
                    st_release_u64(p.flags + blockIdx.x, p.token);
                }
            } else {
                float4 v[EPT];
#pragma unroll
                for (int i = 0; i < EPT; ++i) {
                    const int e = ct + i * 32 * NW;
                    v[i] = e < NE ? *reinterpret_cast<const float4*>(tile + (e >> 5) * L::TS + 4 * (e & 31))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                bool fin_ok = true;
                if (head) {
                    // add the other pieces of this slab, held by the next CTAs, in CTA order.
                    // Lane i of warp 0 watches the token of CTA blockIdx.x + 1 + i (all polls
                    // in flight at once); then every thread loads its elements of every
                    // partial tile at once and adds them in CTA order.
                    const int cl = dec_cta_of_unit(sc.slab * G + G - 1, p.units, p.grid);
                    const int np = cl - (int)blockIdx.x;  // partial tiles to add
                    int ready = 1;
                    if (warp == 0) {
                        const unsigned long long t0 = globaltimer_ns();
                        const unsigned long long lim = g_wait_limit_ns;
                        for (int i0 = 0; i0 < np; i0 += 32) {
                            const int c = (int)blockIdx.x + 1 + i0 + lane;
                            bool seen = i0 + lane >= np;  // lanes past the last piece have nothing to watch
                            for (uint32_t it = 0;; ++it) {
                                if (!seen) seen = ld_acquire_u64(p.flags + c) == p.token;
                                if (__all_sync(0xffffffffu, seen)) break;
                                __nanosleep(32);
                                if ((it & 15u) == 15u && globaltimer_ns() - t0 > lim) {
                                    if (lane == 0) set_status(7u);
                                    ready = 0;
                                    break;
                                }
                            }
                            if (!ready) break;
                        }
                    }
                    fin_ok = named_bar_and(1, 32 * NW, ready) != 0;
                    const float4* base = reinterpret_cast<const float4*>(p.partials);
                    constexpr int NB = EPT >= 8 ? 1 : 8 / EPT;  // partial tiles whose loads are in flight together (32 registers)
#pragma unroll 1
                    for (int c0 = (int)blockIdx.x + 1; fin_ok && c0 <= cl; c0 += NB) {
                        float4 w[NB][EPT];
#pragma unroll
                        for (int r = 0; r < NB; ++r)
#pragma unroll
                            for (int i = 0; i < EPT; ++i) {
                                const int e = ct + i * 32 * NW;
                                if (c0 + r <= cl && e < NE) w[r][i] = __ldcg(base + (size_t)(c0 + r) * (L::PARTIAL_FLOATS / 4) + e);
                            }
#pragma unroll
                        for (int r = 0; r < NB; ++r)
#pragma unroll
                            for (int i = 0; i < EPT; ++i)
                                if (c0 + r <= cl) {
                                    v[i].x += w[r][i].x;
                                    v[i].y += w[r][i].y;
                                    v[i].z += w[r][i].z;
                                    v[i].w += w[r][i].w;
                                }
                    }
                    named_bar_sync(1, 32 * NW);
                    if (fin_ok && warp == 0)
                        for (int c = (int)blockIdx.x + 1 + lane; c <= cl; c += 32) p.flags[c] = 0ull;  // consumed: clear
                }
                if (fin_ok) {
                    // Y: four adjacent columns of one token per element (N % 16 == 0)
#pragma unroll
                    for (int i = 0; i < EPT; ++i) {
                        const int e = ct + i * 32 * NW;
                        const int tok = e >> 5, col = n0 + 4 * (e & 31);
                        if (e < NE && tok < p.M && col < p.N) {
                            const uint2 o = make_uint2((uint32_t)H::to_bits(v[i].x) | ((uint32_t)H::to_bits(v[i].y) << 16),
                                                       (uint32_t)H::to_bits(v[i].z) | ((uint32_t)H::to_bits(v[i].w) << 16));
                            *reinterpret_cast<uint2*>(p.Y + (int64_t)tok * p.N + col) = o;
                        }
                    }
                }
            }
        }
        named_bar_sync(1, 32 * NW);  // the tile is free for the next piece

        // 4. every consumer starts the next piece from zero
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int j = 0; j < MT; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[h][c][j][e] = 0.0f;
    }
}

}  // namespace qg
