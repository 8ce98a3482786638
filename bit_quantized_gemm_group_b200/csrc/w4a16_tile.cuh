// w4a16_tile.cuh -- prefill-shape W4A16 fused dequant-GEMM on the tcgen05 tensor cores
// (M >= kTcMinM tokens, bf16 activations).
//
//   Y[m][n] = sum_k X[m][k] W[k][n],   W[k][n] = (q[k][n] - z[g][n]) s[g][n],  g = k / 128
// ("AI Infra guide, ch.4 Quantization" sec. 3.1 weight-only INT4, sec. 3.5 fused
// INT4 x FP16 kernel: dequantize in registers, multiply on the tensor cores).
//
// Swap-AB with the weights in tensor memory.  A tile is 128 weight columns (the MMA's
// M) by 256 tokens (its N); the MMA computes D[n][m] = sum_k W[k][n] X[m][k] with
//   A = the dequantized weight tile, written to TMEM by the dequant warps (tcgen05.st;
//       lane = column n, each 32-bit cell two consecutive k as bf16),
//   B = the activation tile [256 tokens][64 k], K-major with 128-byte swizzle, as TMA
//       writes it,
//   D = fp32 in TMEM, 256 columns (one per token) x 128 lanes.
// The dequantized weights never touch shared memory, so shared memory holds only what
// TMA brings (activations and packed words): six stages of 36 KB, enough bytes in
// flight to cover the load latency of the activation re-reads.  Each MMA is N = 256,
// so one issuing thread keeps the tensor core busy.
//
// Dequant: a packed word holds 8 consecutive k of column n (nibbles low first).  OR-ing
// a nibble pair into the exponent field of a bf16 pair gives exactly 128 + q; a packed
// subtract of 128 + z and a multiply by s give (q - z) s rounded to bf16 (the operand
// type of the tensor core); byte permutes put the pairs in natural k order.
//
// Roles (640 threads): warp 0 issues TMA; warp 1 owns tensor memory and issues the
// MMAs; warps 4-11 run the epilogue (warp w: TMEM lanes 32 (w % 4), tokens
// 128 ((w - 4) / 4) .. + 127); warps 12-19 dequantize (warp w: TMEM lanes 32 (w % 4),
// words 4 ((w - 12) / 4) .. + 3 of the k-block).  The persistent grid walks the tiles
// with the token index fastest, so CTAs running together share weight tiles in L2.
#pragma once
#include "common.cuh"
#include "tc_gemm.cuh"

namespace qg {

struct W4TileCfg {
    static constexpr int BW = 128;  // weight columns per tile (MMA M)
    static constexpr int BT = 256;  // tokens per tile (MMA N)
    static constexpr int BK = 64;   // k per stage
    static constexpr int X_BYTES = BT * BK * 2;      // 32 KB
    static constexpr int RAW_BYTES = (BK / 8) * BW * 4;  // 4 KB: [8 words][128 columns]
    static constexpr int STAGE = X_BYTES + RAW_BYTES;
    static constexpr int ST = 6;
    static constexpr int AS = 8;      // TMEM A slots of 32 columns (one k-block)
    static constexpr int A_COL0 = BT; // D in columns [0, 256), A slots after it
    static constexpr int TMEM_COLS = 512;
    static_assert(A_COL0 + AS * 32 <= TMEM_COLS, "tensor memory budget");
    static constexpr int EPI = 8, DQ = 8;
    static constexpr int THREADS = 32 * (4 + EPI + DQ);
    static constexpr int BAR_OFF = ST * STAGE;
    // full[ST] empty[ST] afull[AS] aempty[AS] tfull tempty done
    static constexpr int NBAR = 2 * ST + 2 * AS + 3;
    static constexpr int TOTAL = BAR_OFF + NBAR * 8 + 16 + 1024;
};

struct W4TileParams {
    const uint16_t* scales;  // fp16 [K/128][N]
    const uint8_t* zeros;    // u8 [K/128][N]
    uint16_t* Y;             // bf16 [M][N]
    int M, K, N;
    int t_tiles, w_tiles;    // token tiles (256), weight tiles (128)
};

__global__ void __launch_bounds__(W4TileCfg::THREADS, 1)
    w4a16_tile_kernel(const W4TileParams p, const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_w)
{
    using C = W4TileCfg;
    constexpr int ST = C::ST, AS = C::AS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* empty = full + ST;
    uint64_t* afull = empty + ST;
    uint64_t* aempty = afull + AS;
    uint64_t* tfull = aempty + AS;
    uint64_t* tempty = tfull + 1;
    uint64_t* done = tempty + 1;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = p.K / C::BK;
    const int num_tiles = p.t_tiles * p.w_tiles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + C::DQ);  // the MMA commit and the dequant warps
        }
        for (int i = 0; i < AS; ++i) {
            mbar_init(&afull[i], 32 * C::DQ);
            mbar_init(&aempty[i], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 32 * C::EPI);
        mbar_init(done, 1);
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
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_w);
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % p.t_tiles) * C::BT, n0 = (tile / p.t_tiles) * C::BW;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % ST;
                    if (!mbar_wait(&empty[s], ((it / ST) & 1) ^ 1)) { ok = false; break; }
                    uint8_t* st = smem + s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(&tm_x, &full[s], st, kb * C::BK, m0);
                    tma_load_2d(&tm_w, &full[s], st + C::X_BYTES, n0, kb * (C::BK / 8));
                }
            }
            // every copy still in flight lands before the CTA exits
            for (int j = it - ST > 0 ? it - ST : 0; j < it; ++j) mbar_wait(&full[j % ST], (j / ST) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(C::BT);
            int it = 0, li = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++li) {
                if (!mbar_wait(tempty, (li & 1) ^ 1)) break;  // the epilogue has drained D
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % ST, a = it % AS;
                    if (!mbar_wait(&full[s], (it / ST) & 1) || !mbar_wait(&afull[a], (it / AS) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xs = smem_u32(smem + s * C::STAGE);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_f16_ts(tmem, tmem + C::A_COL0 + 32 * a + 8 * kk, smem_desc(xs + 32 * kk, 16, 1024, 2), idesc,
                                   (kb | kk) != 0);
                    mma_commit(&aempty[a]);
                    mma_commit(&empty[s]);
                    issued = true;
                }
                if (ok) mma_commit(tfull);
            }
            if (issued) {  // every MMA has completed before tensor memory is released
                mma_commit(done);
                mbar_wait(done, 0);
            }
        }
    } else if (warp < 4) {
        // warps 2, 3: no role
    } else if (warp < 4 + C::EPI) {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3, th = (warp - 4) >> 2;  // TMEM lane quarter, token half
        int li = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++li) {
            const int m0 = (tile % p.t_tiles) * C::BT, n0 = (tile / p.t_tiles) * C::BW;
            const int n = n0 + 32 * q + lane;
            if (!warp_wait(tfull, li & 1)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const int t0 = 128 * th + 32 * c;  // tokens t0 .. t0 + 31 of the tile
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + t0, r);
                tmem_ld_wait();
                const int nt = min(32, p.M - m0 - t0);
                if ((p.N & 1) == 0) {
                    // 2 x 2 transpose between lane pairs, then one 4-byte store of two
                    // adjacent columns per lane: the even lane writes token t, the odd
                    // lane token t + 1 (half the store instructions of 2-byte stores)
                    const bool even = (lane & 1) == 0;
                    const int c0 = even ? n : n - 1;
#pragma unroll
                    for (int t = 0; t < 32; t += 2) {
                        const float a = __uint_as_float(r[t]), b = __uint_as_float(r[t + 1]);
                        const float recv = __shfl_xor_sync(0xffffffffu, even ? b : a, 1);
                        const int row = t + (even ? 0 : 1);
                        const uint32_t v = even ? pack_bf16x2_rn(a, recv) : pack_bf16x2_rn(recv, b);
                        if (row < nt && c0 + 1 < p.N)
                            *reinterpret_cast<uint32_t*>(p.Y + (int64_t)(m0 + t0 + row) * p.N + c0) = v;
                    }
                } else if (n < p.N) {  // odd N: rows are not 4-byte aligned
                    uint16_t* y = p.Y + (int64_t)(m0 + t0) * p.N + n;
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (t < nt) y[(int64_t)t * p.N] = f32_to_bf16_bits(__uint_as_float(r[t]));
                }
            }
            tc_fence_before();
            mbar_arrive(tempty);
        }
    } else {
        // ------------------------------ dequant warps ------------------------------
        const int q = (warp - 4 - C::EPI) & 3, kh = (warp - 4 - C::EPI) >> 2;  // lane quarter, word half
        const int col = 32 * q + lane;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int n = (tile / p.t_tiles) * C::BW + col;
            // per-column scale and zero, fetched one group ahead of their use
            uint16_t s_cur = 0, s_nxt = 0;
            uint8_t z_cur = 0, z_nxt = 0;
            if (n < p.N) {
                s_cur = __ldg(p.scales + n);
                z_cur = __ldg(p.zeros + n);
                if (KB > 2) {
                    s_nxt = __ldg(p.scales + (int64_t)p.N + n);
                    z_nxt = __ldg(p.zeros + (int64_t)p.N + n);
                }
            }
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % ST, a = it % AS;
                if (kb > 0 && (kb & 1) == 0) {  // a new group starts: rotate and prefetch the next
                    s_cur = s_nxt;
                    z_cur = z_nxt;
                    const int gn = (kb >> 1) + 1;
                    if (n < p.N && 2 * gn < KB) {
                        s_nxt = __ldg(p.scales + (int64_t)gn * p.N + n);
                        z_nxt = __ldg(p.zeros + (int64_t)gn * p.N + n);
                    }
                }
                const float sv = __half2float(__ushort_as_half(s_cur));
                const uint32_t s2 = pack_bf16x2_rn(sv, sv);
                const uint32_t z2 = 0x43004300u | ((uint32_t)z_cur * 0x00010001u);  // 128 + z, exact
                if (!mbar_wait(&full[s], (it / ST) & 1)) { ok = false; break; }
                const uint32_t* raw = reinterpret_cast<const uint32_t*>(smem + s * C::STAGE + C::X_BYTES);
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = raw[(4 * kh + i) * 128 + col];
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);  // packed words consumed
                uint32_t cell[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t R[4];  // (k r, k r + 4) of the word, as (q - z) s
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        R[r] = bf16x2_mul(bf16x2_sub(lop3_and_or(w[i] >> (4 * r), 0x000F000Fu, 0x43004300u), z2), s2);
                    cell[4 * i + 0] = prmt(R[0], R[1], 0x5410);  // k 0, 1
                    cell[4 * i + 1] = prmt(R[2], R[3], 0x5410);  // k 2, 3
                    cell[4 * i + 2] = prmt(R[0], R[1], 0x7632);  // k 4, 5
                    cell[4 * i + 3] = prmt(R[2], R[3], 0x7632);  // k 6, 7
                }
                if (!mbar_wait(&aempty[a], ((it / AS) & 1) ^ 1)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x16(tmem + ((uint32_t)(32 * q) << 16) + C::A_COL0 + 32 * a + 16 * kh, cell);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&afull[a]);
            }
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
