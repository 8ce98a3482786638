// w4a16_decode.cuh -- decode-shape W4A16 fused dequant-GEMM (M <= 32 per launch).
//
//   Y[m][n] = sum_k X[m][k] (q[k][n] - z[g][n]) s[g][n],   g = k / 128
// ("AI Infra guide, ch.4 Quantization" sec. 3.1 weight-only INT4, sec. 3.5 fused
// INT4 x FP16 kernel; group-wise scale and zero: "LLM inference cost: W8A8/W4A8 ..."
// sec. 2.2).  Decode is a weight stream: the design keeps HBM busy and the ALU cost
// per weight small.
//
// Work split (stream-K).  The N columns form slabs of 128; one unit is one group
// (128 k) of one slab.  The persistent grid (one CTA per SM) divides the
// nslabs x G units into equal contiguous ranges, so every SM streams the same
// number of bytes.  A CTA's range is a list of slab pieces: a piece that covers a
// whole slab writes Y directly; a partial piece writes its fp32 tile to the workspace
// (slot 0 for the CTA's first piece, 1 for its last).  The follow-up kernel
// `w4a16_decode_fixup_kernel` sums the pieces of every split slab in CTA order
// (deterministic; no atomics, no counters) and writes Y.
//
// Data movement.  One producer thread streams the packed words (16 rows of the [K/8][N]
// matrix x 128 columns per group, 128-byte swizzled), fp16 scales, u8 zeros and the
// activation tiles into a ring of shared-memory stages with TMA; a stage holds up to
// four groups of one slab and, when full, arrives in four bulk copies (DecodeMaps).
// Consumer warp (wn, wg, ws) takes columns 64wn..64wn+63 of group wg of each stage and
// the ws-th share of its four 32-k steps (WS = 1 or 2 warps per group).
//
// Math.  Swap-AB mma.sync (weights are the m16 operand, up to 32 tokens are n8
// tiles).  A lane's 128-bit read gives 4 columns x 8 k; OR-ing a nibble pair into
// the exponent field of a bf16 (fp16) pair yields exactly 128 + q (1024 + q) with
// one LOP3, so the MMA accumulates D = sum (128 + q) x per group.  The zero point and
// scale are applied once per group and output element:
//     acc += s * (D - (128 + z) * sum_{k} x)
// where sum x comes from one extra MMA tile whose A operand is all ones, already in
// the accumulator layout (the correction is linear, so each warp applies it to its
// own share of the steps).  Inside a 32-k step the k order is permuted so that a
// lane's own word feeds its fragment slots; the activation pairs get the same
// permutation with byte permutes.  Shared-memory rows are visited in the order
// 0,2,4,6 | 1,3,5,7 | 8,... so the eight lanes of each 128-bit access phase hit eight
// different 16-byte bank groups under the 128-byte swizzle.
//
// Programmatic dependent launch: the kernel lets the next grid launch at once; the
// producer requests the first ring-full of weights before waiting for the previous
// grid (griddepcontrol.wait), and nothing that depends on it (X, Y, the workspace)
// is touched before that wait.
#pragma once
#include "common.cuh"
#include "w4a16_skinny.cuh"

namespace qg {

struct DecodeParams {
    const uint16_t* X;
    uint16_t* Y;
    float* partials;  // [grid][2][MP][128]
    int M, K, N;
    int G, nslabs, units, grid;
};

constexpr int kDecBN = 128;               // columns per slab
constexpr int kDecGroupsPerStage = 4;
constexpr int kDecGroupW = 16 * 128 * 4;  // packed words of one group: 16 rows x 128 columns x 4 B
// (a stage holds them as [column block of 32][group][16 rows][128 B], 128-byte swizzled)
constexpr int kDecScaleOff = 4 * kDecGroupW;
constexpr int kDecZeroOff = kDecScaleOff + 4 * 256;
constexpr int kDecXOff = kDecZeroOff + 4 * 128 + 512;  // 1 KB aligned
constexpr int kMaxPieces = 160;           // grid cap: pieces of one slab (one per CTA at most)

QG_DEV_INLINE int dec_first_unit(int c, int units, int grid) { return (int)((int64_t)c * units / grid); }

// CTA holding unit u of the static split
QG_DEV_INLINE int dec_cta_of_unit(int u, int units, int grid)
{
    int c = (int)((int64_t)u * grid / units);
    while (c > 0 && dec_first_unit(c, units, grid) > u) --c;
    while (dec_first_unit(c + 1, units, grid) <= u) ++c;
    return c;
}

// Stage: 4 groups x {packed words 8 KB, fp16 scales 256 B, u8 zeros 128 B, X tile
// MP tokens x 128 k bf16 as two 128-byte-swizzled boxes of 64 k}.
template <int MT, int ST, int WS>
struct DecodeSmem {
    static constexpr int MP = 8 * MT;
    static constexpr int XG = MP * 256;  // X bytes per group
    static constexpr int STAGE = kDecXOff + 4 * XG;
    static constexpr int RS = kDecBN + 8;  // padded row of the [token][column] reduction tile
    static constexpr int NRED = 4 * WS;    // warps adding into one column half
    static constexpr int RED = NRED * MP * RS * 4;
    static constexpr int TOTAL = ST * STAGE + RED + 2 * ST * 8 + 1024;
    static constexpr uint32_t GROUP_TX = kDecGroupW + 256 + 128 + XG;
    static constexpr int NC = 8 * WS;      // consumer warps
    static constexpr int THREADS = 32 * NC + 128;
};

// Tensor maps.  A full stage (four groups of one slab) comes in four copies: the
// packed words as four 32-column x 64-row boxes (128-byte swizzle), the scales and zeros
// as 4-row boxes, and the activation tile as one 3-D box {64 k, MP rows, 8 halves}
// that lands as [group][half][row][128 B].  A thread's bulk copies are issued one after
// another at a cost of roughly a hundred cycles each, so few large copies keep the
// producer ahead of the weight stream.  Stages of fewer groups (a piece's last) use
// one-group boxes into the same layout.
struct DecodeMaps {
    CUtensorMap w4, w1;  // packed words: {32 columns, 64 | 16 rows}
    CUtensorMap s4, s1;  // fp16 scales:  {128 columns, 4 | 1 groups}
    CUtensorMap z4, z1;  // u8 zeros:     {128 columns, 4 | 1 groups}
    CUtensorMap x4, x1;  // activations:  {64 k, MP rows, 8 | 2 halves}
};

template <int MT, bool BF16, int ST, int WS>
__global__ void __launch_bounds__(DecodeSmem<MT, ST, WS>::THREADS, 1)
    w4a16_decode_kernel(const DecodeParams p, const __grid_constant__ DecodeMaps maps)
{
    using H = HalfOps<BF16>;
    using L = DecodeSmem<MT, ST, WS>;
    constexpr int MP = 8 * MT;
    constexpr int NC = L::NC;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* red = reinterpret_cast<float*>(smem + ST * L::STAGE);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * L::STAGE + L::RED);
    uint64_t* empty = full + ST;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.G;
    const int u0 = dec_first_unit(blockIdx.x, p.units, p.grid), u1 = dec_first_unit(blockIdx.x + 1, p.units, p.grid);

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], NC);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp >= NC) {
        // ---------------- producer warpgroup (one thread issues TMA) ----------------
        // Register split (setmaxnreg works per warpgroup): this warpgroup keeps few
        // registers and hands the rest to the consumer warpgroups.
        if constexpr (WS == 1) asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");   // 384 x 168 at launch
        else asm volatile("setmaxnreg.dec.sync.aligned.u32 24;");                    // 640 x 96 at launch
        if (warp == NC && lane == 0) {
            tma_prefetch_desc(&maps.w4);
            tma_prefetch_desc(&maps.s4);
            tma_prefetch_desc(&maps.z4);
            tma_prefetch_desc(&maps.x4);
            // activation tiles of a stage: one 3-D box for four groups, else per group
            auto load_x = [&](uint64_t* bar, uint8_t* st, int g0, int ng) {
                if (ng == kDecGroupsPerStage)
                    tma_load_3d(&maps.x4, bar, st + kDecXOff, 0, 0, 2 * g0);
                else
                    for (int i = 0; i < ng; ++i) tma_load_3d(&maps.x1, bar, st + kDecXOff + i * L::XG, 0, 0, 2 * (g0 + i));
            };
            // Weights, scales and zeros do not depend on the previous grid: the first
            // ring-full of them is requested before waiting for it; X after.
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool waited = false, ok = true;
            int pend_g0[ST], pend_ng[ST];
            for (int u = u0; u < u1 && ok;) {
                const int slab = u / G, ga = u % G;
                const int gb = min(G, ga + (u1 - u));
                for (int g0 = ga; g0 < gb; g0 += kDecGroupsPerStage) {
                    const int ng = min(kDecGroupsPerStage, gb - g0);
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)ng * L::GROUP_TX);
                    uint8_t* st = ring + stage * L::STAGE;
                    const int x = slab * kDecBN;
                    if (ng == kDecGroupsPerStage) {
#pragma unroll
                        for (int b = 0; b < 4; ++b) tma_load_2d(&maps.w4, &full[stage], st + b * 4 * 2048, x + 32 * b, 16 * g0);
                        tma_load_2d(&maps.s4, &full[stage], st + kDecScaleOff, x, g0);
                        tma_load_2d(&maps.z4, &full[stage], st + kDecZeroOff, x, g0);
                    } else {
                        for (int i = 0; i < ng; ++i) {
#pragma unroll
                            for (int b = 0; b < 4; ++b)
                                tma_load_2d(&maps.w1, &full[stage], st + b * 4 * 2048 + i * 2048, x + 32 * b, 16 * (g0 + i));
                            tma_load_2d(&maps.s1, &full[stage], st + kDecScaleOff + i * 256, x, g0 + i);
                            tma_load_2d(&maps.z1, &full[stage], st + kDecZeroOff + i * 128, x, g0 + i);
                        }
                    }
                    if (!waited && issued < ST) {
                        pend_g0[issued] = g0;
                        pend_ng[issued] = ng;
                    }
                    if (!waited && (issued + 1 == ST || (g0 + kDecGroupsPerStage >= gb && u + (gb - ga) >= u1))) {
                        // ring full (or schedule done): now wait for the previous grid, then load X
                        asm volatile("griddepcontrol.wait;" ::: "memory");
                        waited = true;
                        for (int j = 0; j <= issued; ++j) load_x(&full[j], ring + j * L::STAGE, pend_g0[j], pend_ng[j]);
                    } else if (waited) {
                        load_x(&full[stage], st, g0, ng);
                    }
                    ++issued;
                    if (++stage == ST) { stage = 0; phase ^= 1; }
                }
                u += gb - ga;
            }
            if (!waited) {
                // gave up inside the first ring-full: complete the stages requested so
                // far, so that every copy in flight can land
                asm volatile("griddepcontrol.wait;" ::: "memory");
                for (int j = 0; j < issued; ++j) load_x(&full[j], ring + j * L::STAGE, pend_g0[j], pend_ng[j]);
            }
            // every copy still in flight lands before the CTA exits
            for (int j = issued - ST > 0 ? issued - ST : 0; j < issued; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        }
        return;
    }

    // ---------------- consumers ----------------
    if constexpr (WS == 1) asm volatile("setmaxnreg.inc.sync.aligned.u32 232;");
    else asm volatile("setmaxnreg.inc.sync.aligned.u32 112;");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int wn = warp & 1, wg = (warp >> 1) & 3, ws = warp >> 3;
    constexpr int SPW = 4 / WS;  // 32-k steps per warp per group
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
    bool first_piece = true;
    // After a wait gives up (status already recorded) the warp keeps walking the same
    // schedule without waiting or computing, so that every named barrier still sees
    // all consumer threads; nothing is written to global memory after that.
    for (int u = u0; u < u1;) {
        const int slab = u / G, ga = u % G;
        const int gb = min(G, ga + (u1 - u));
        const int n0 = slab * kDecBN;
        for (int g0 = ga; g0 < gb; g0 += kDecGroupsPerStage) {
            const int ng = min(kDecGroupsPerStage, gb - g0);
            if (ok && !mbar_wait_backoff(&full[stage], phase)) ok = false;
            const uint8_t* st = ring + stage * L::STAGE;
            if (ok && wg < ng) {
                // per-column scale and (128 + z) of the lane's 8 columns
                float sc[2][4], zc[2][4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = 64 * wn + 32 * h + 4 * g8;
                    const uint2 s4 = *reinterpret_cast<const uint2*>(st + kDecScaleOff + wg * 256 + col * 2);
                    const uint32_t z4 = *reinterpret_cast<const uint32_t*>(st + kDecZeroOff + wg * 128 + col);
                    const uint32_t sw[2] = {s4.x, s4.y};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        sc[h][c] = __half2float(__ushort_as_half((unsigned short)(sw[c >> 1] >> (16 * (c & 1)))));
                        zc[h][c] = H::BIAS + (float)((z4 >> (8 * c)) & 0xFFu);
                    }
                }
                float D[2][2][MT][4], Dx[MT][4];
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
                const uint8_t* wbase = st + wg * 2048;  // column block b of group wg at b * 8 KB + wg * 2 KB
                const uint8_t* xg = st + kDecXOff + wg * L::XG;
#pragma unroll
                for (int si = 0; si < SPW; ++si) {
                    const int s = ws * SPW + si;
                    const int row = 8 * (s >> 1) + 2 * t4 + (s & 1);  // kb row within the group
                    uint4 wv[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        wv[h] = *reinterpret_cast<const uint4*>(wbase + (2 * wn + h) * 8192 + row * 128 +
                                                                ((g8 ^ (row & 7)) << 4));
                    uint32_t xb[MT][4];
                    const uint8_t* xs = xg + (row >> 3) * (L::XG / 2);
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const int tok = 8 * j + g8;  // rows >= M are zero (TMA fill)
                        const uint4 xv = *reinterpret_cast<const uint4*>(xs + tok * 128 + (((row & 7) ^ (tok & 7)) << 4));
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
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int r = 0; r < 4; ++r) R[c][r] = lop3_and_or(w[c] >> (4 * r), 0x000F000Fu, H::MAGIC);
#pragma unroll
                        for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                            for (int j = 0; j < MT; ++j) {
                                mma_16816<BF16>(D[h][cp][j], R[2 * cp][0], R[2 * cp + 1][0], R[2 * cp][1],
                                                R[2 * cp + 1][1], xb[j][0], xb[j][1]);
                                mma_16816<BF16>(D[h][cp][j], R[2 * cp][2], R[2 * cp + 1][2], R[2 * cp][3],
                                                R[2 * cp + 1][3], xb[j][2], xb[j][3]);
                            }
                    }
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        mma_16816<BF16>(Dx[j], ONE, ONE, ONE, ONE, xb[j][0], xb[j][1]);
                        mma_16816<BF16>(Dx[j], ONE, ONE, ONE, ONE, xb[j][2], xb[j][3]);
                    }
                }
                // group epilogue (this warp's steps): acc += s * (D - (128 + z) * sum x)
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                        for (int j = 0; j < MT; ++j)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = 2 * cp + (e >> 1);
                                const float xs = Dx[j][e & 1];
                                acc[h][cp][j][e] = fmaf(sc[h][c], fmaf(-zc[h][c], xs, D[h][cp][j][e]), acc[h][cp][j][e]);
                            }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == ST) { stage = 0; phase ^= 1; }
        }

        // ---------------- piece end: reduce the group-warps of each column half ----------------
        // Reduction tile layout [token][column] with a padded row, so that the fragment
        // stores are at most 2-way conflicted and every later pass reads consecutive words.
        constexpr int RS = L::RS;
        float* myred = red + (size_t)(wg * WS + ws) * MP * RS;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int cp = 0; cp < 2; ++cp)
#pragma unroll
                for (int j = 0; j < MT; ++j) {
                    const int nl = 64 * wn + 32 * h + 4 * g8 + 2 * cp;
                    const int tk = 8 * j + 2 * t4;
                    *reinterpret_cast<float2*>(myred + tk * RS + nl) = make_float2(acc[h][cp][j][0], acc[h][cp][j][2]);
                    *reinterpret_cast<float2*>(myred + (tk + 1) * RS + nl) = make_float2(acc[h][cp][j][1], acc[h][cp][j][3]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[h][cp][j][e] = 0.0f;
                }
        named_bar_sync(1, 32 * NC);
        const int mrows = min(p.M, MP);
        // any warp that gave up makes the whole CTA skip its global writes
        const int all_ok = named_bar_and(1, 32 * NC, ok);
        if (!all_ok) {
            ok = false;
        } else {
            const bool whole = ga == 0 && gb == G;
            const int nvalid = min(kDecBN, p.N - n0);
            float* mine = p.partials + ((size_t)blockIdx.x * 2 + (first_piece ? 0 : 1)) * MP * kDecBN;
            // sum the group-warps, 4 consecutive columns per thread step; write Y (whole
            // slab) or this piece's partial tile [token][128] (split slab)
            for (int e = threadIdx.x; e < mrows * (kDecBN / 4); e += 32 * NC) {
                const int tok = e / (kDecBN / 4), c4 = 4 * (e % (kDecBN / 4));
                float4 v = *reinterpret_cast<const float4*>(red + tok * RS + c4);
#pragma unroll
                for (int q = 1; q < L::NRED; ++q) {
                    const float4 w = *reinterpret_cast<const float4*>(red + (size_t)q * MP * RS + tok * RS + c4);
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                if (whole) {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        if (c4 + r < nvalid) p.Y[(int64_t)tok * p.N + n0 + c4 + r] = H::to_bits(vv[r]);
                } else {
                    *reinterpret_cast<float4*>(mine + tok * kDecBN + c4) = v;
                }
            }
        }
        named_bar_sync(1, 32 * NC);
        first_piece = false;
        u += gb - ga;
    }
}

// Sums the pieces of every slab that the decode grid split between CTAs, in CTA order,
// and writes Y.  One CTA per slab; slabs held by one CTA were written directly.
template <bool BF16>
__global__ void __launch_bounds__(256) w4a16_decode_fixup_kernel(const DecodeParams p, int MP)
{
    using H = HalfOps<BF16>;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int slab = blockIdx.x;
    const int G = p.G;
    const int cf = dec_cta_of_unit(slab * G, p.units, p.grid);
    const int cl = dec_cta_of_unit(slab * G + G - 1, p.units, p.grid);
    if (cf == cl) return;  // the whole slab was one piece: written by the decode kernel
    __shared__ int off[kMaxPieces];
    for (int c = cf + threadIdx.x; c <= cl; c += blockDim.x) {
        const int sl = dec_first_unit(c, p.units, p.grid) >= slab * G ? 0 : 1;  // first piece of CTA c?
        off[c - cf] = (c * 2 + sl) * MP * kDecBN;
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the decode grid's partial tiles are complete
    const int np = cl - cf + 1;
    const int n0 = slab * kDecBN;
    const int nvalid = min(kDecBN, p.N - n0);
    const int mrows = min(p.M, MP);
    for (int e = threadIdx.x; e < mrows * (kDecBN / 4); e += blockDim.x) {
        const int tok = e / (kDecBN / 4), c4 = 4 * (e % (kDecBN / 4));
        const int o = tok * kDecBN + c4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        int i = 0;
        for (; i + 4 <= np; i += 4) {  // four independent loads in flight, summed in piece order
            float4 a[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = __ldcg(reinterpret_cast<const float4*>(p.partials + off[i + r] + o));
#pragma unroll
            for (int r = 0; r < 4; ++r) { v.x += a[r].x; v.y += a[r].y; v.z += a[r].z; v.w += a[r].w; }
        }
        for (; i < np; ++i) {
            const float4 a = __ldcg(reinterpret_cast<const float4*>(p.partials + off[i] + o));
            v.x += a.x; v.y += a.y; v.z += a.z; v.w += a.w;
        }
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
            if (c4 + r < nvalid) p.Y[(int64_t)tok * p.N + n0 + c4 + r] = H::to_bits(vv[r]);
    }
}

}  // namespace qg
