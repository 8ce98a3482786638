// gptq_blocked.cuh -- GPTQ in its blocked, Cholesky form (the fast offline path).
//
// "Quantization & Flash Attention -- LLM inference optimization (2)", sec. 3.1-3.3:
// rows of W are rounded in order and each row's rounding error is spread over the rows
// not yet rounded through the inverse Hessian.  After rows 0..k-1 have been eliminated,
// row k of the remaining inverse divided by the square root of its diagonal is row k of
// the upper Cholesky factor U of H^-1 (H^-1 = U^T U).  So with
//     err_k = (w_k - deq(q_k)) / U[k][k],      w_j -= err_k U[k][j]   (j > k)
// every row is compensated exactly as in the sequential definition, and U is computed
// once.  The updates of a block of rows (one quantization group) are applied inside the
// block as the rows are rounded; the rows after the block receive all of them at once,
// one GEMM per block:  W[after] -= U[block, after]^T Err[block].
//
// U without forming H^-1: H is reversed (Hr = J H J, J the index reversal), Hr = Lr Lr^T
// (lower Cholesky), and then H = V V^T with V = J Lr J upper, so H^-1 = V^-T V^-1 and
//     U = V^-1 = J Lr^-1 J,   U[i][j] = Lr^-1[K-1-i][K-1-j].
// Steps, all binary64:
//   Xr[m][i] = x[m][K-1-i]; Hr = (2/Mc) Xr^T Xr (lower); + lambda on the diagonal;
//   Lr by a right-looking blocked Cholesky (64-wide panels: the diagonal block factored
//   and inverted in one CTA, the panel below multiplied by that inverse, the trailing
//   lower triangle updated by a GEMM);
//   Lr^-1 by block rows: row block i = -D_i (Lr[i, <i] Lr^-1[<i, <i]) beside D_i, where
//   D_i is the inverse of the i-th diagonal block kept from the factorization;
//   then the blocks of rows of W as above, reading U through the reversal.
// The sums run in another order than the sequential definition's, so codes may differ
// where a compensated weight sits within rounding noise of a rounding boundary; the
// scale and zero of a group come from its compensated weights exactly as there.
#pragma once
#include "common.cuh"

namespace qg {

constexpr int kCholNb = 64;  // panel width of the factorization and of the inverse

// C[i][j] = alpha sum_k A(i, k) B(k, j) + beta C[i][j], A(i, k) = A[i a_i + k a_k],
// B(k, j) = B[k b_k + j b_j] (signed strides: reversed views need no copy).
// lower_c: only i >= j is computed and written (tiles wholly above skip).
// lower_b: B(k, j) = 0 for k < j, so a column tile starts its k loop at its first column.
struct DgemmArgs {
    int M, N, Kd;
    double alpha, beta;
    const double* A;
    int64_t a_i, a_k;
    const double* B;
    int64_t b_k, b_j;
    double* C;
    int64_t ldc;
    int lower_c, lower_b;
};

template <int BM, int BN>
__global__ void __launch_bounds__(256) dgemm_strided_kernel(const DgemmArgs a)
{
    constexpr int BK = 16, TM = BM / 16, TN = BN / 16;
    __shared__ double As[BK][BM + 1];
    __shared__ double Bs[BK][BN + 1];
    const int i0 = blockIdx.y * BM, j0 = blockIdx.x * BN;
    if (a.lower_c && j0 > i0 + BM - 1) return;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const bool a_icont = a.a_i == 1 || a.a_i == -1;
    const bool b_jcont = a.b_j == 1 || a.b_j == -1;
    double acc[TM][TN];
#pragma unroll
    for (int r = 0; r < TM; ++r)
#pragma unroll
        for (int c = 0; c < TN; ++c) acc[r][c] = 0.0;
    const int kbeg = a.lower_b ? (j0 / BK) * BK : 0;
    for (int k0 = kbeg; k0 < a.Kd; k0 += BK) {
#pragma unroll
        for (int e = 0; e < BM * BK / 256; ++e) {
            const int idx = tid + 256 * e;
            const int i = a_icont ? idx % BM : idx / BK, k = a_icont ? idx / BM : idx % BK;
            const int gi = i0 + i, gk = k0 + k;
            As[k][i] = (gi < a.M && gk < a.Kd) ? a.A[(int64_t)gi * a.a_i + (int64_t)gk * a.a_k] : 0.0;
        }
#pragma unroll
        for (int e = 0; e < BN * BK / 256; ++e) {
            const int idx = tid + 256 * e;
            const int j = b_jcont ? idx % BN : idx / BK, k = b_jcont ? idx / BN : idx % BK;
            const int gj = j0 + j, gk = k0 + k;
            Bs[k][j] = (gj < a.N && gk < a.Kd) ? a.B[(int64_t)gk * a.b_k + (int64_t)gj * a.b_j] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            double av[TM], bv[TN];
#pragma unroll
            for (int r = 0; r < TM; ++r) av[r] = As[kk][ty + 16 * r];
#pragma unroll
            for (int c = 0; c < TN; ++c) bv[c] = Bs[kk][tx + 16 * c];
#pragma unroll
            for (int r = 0; r < TM; ++r)
#pragma unroll
                for (int c = 0; c < TN; ++c) acc[r][c] = fma(av[r], bv[c], acc[r][c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < TM; ++r)
#pragma unroll
        for (int c = 0; c < TN; ++c) {
            const int i = i0 + ty + 16 * r, j = j0 + tx + 16 * c;
            if (i < a.M && j < a.N && (!a.lower_c || i >= j)) {
                double* cp = a.C + (int64_t)i * a.ldc + j;
                *cp = a.beta != 0.0 ? fma(a.alpha, acc[r][c], a.beta * *cp) : a.alpha * acc[r][c];
            }
        }
}

// Xr[m][i] = (double)x[m][K-1-i]
__global__ void __launch_bounds__(256) gptq_xrev_kernel(const uint16_t* __restrict__ X, int Mc, int K,
                                                        double* __restrict__ Xr)
{
    const int64_t total = (int64_t)Mc * K;
    for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = t / K;
        const int i = (int)(t - m * K);
        Xr[t] = (double)bf16_bits_to_f32(__ldg(X + m * K + (K - 1 - i)));
    }
}

// Panel p: the diagonal block A[p..p+nb)[p..p+nb) factored in place (lower), and its
// inverse written to Dinv[p/64] (64 x 64, zeros above the diagonal).  A pivot that is
// not positive is recorded (QG_ERR_RANGE) and replaced by 1 so the rest stays finite.
__global__ void __launch_bounds__(256) chol_diag_kernel(double* __restrict__ A, int K, int p, int nb,
                                                        double* __restrict__ Dinv)
{
    __shared__ double S[kCholNb][kCholNb + 1];
    const int tid = threadIdx.x;
    for (int e = tid; e < kCholNb * kCholNb; e += 256) {
        const int r = e / kCholNb, c = e % kCholNb;
        S[r][c] = (r < nb && c <= r) ? A[(int64_t)(p + r) * K + p + c] : 0.0;
    }
    __syncthreads();
    for (int c = 0; c < nb; ++c) {
        if (tid == 0) {
            double piv = S[c][c];
            if (!(piv > 0.0)) {
                set_status(6u);
                piv = 1.0;
            }
            S[c][c] = sqrt(piv);
        }
        __syncthreads();
        const double d = S[c][c];
        for (int r = c + 1 + tid; r < nb; r += 256) S[r][c] /= d;
        __syncthreads();
        const int w = nb - c - 1;
        for (int e = tid; e < w * w; e += 256) {
            const int r = c + 1 + e / w, s = c + 1 + e % w;
            if (s <= r) S[r][s] -= S[r][c] * S[s][c];
        }
        __syncthreads();
    }
    // inverse of the factor, one column j per thread: L y = e_j by forward substitution
    // (y[q] = 0 for q < j; rows and columns past nb are 0)
    double* D = Dinv + (int64_t)(p / kCholNb) * kCholNb * kCholNb;
    if (tid < kCholNb) {
        const int j = tid;
        double y[kCholNb];
#pragma unroll
        for (int r = 0; r < kCholNb; ++r) {
            double v = 0.0;
            if (r < nb && r == j) {
                v = 1.0 / S[r][r];
            } else if (r < nb && r > j) {
                double acc = 0.0;
#pragma unroll
                for (int q = 0; q < r; ++q) acc = fma(S[r][q], y[q], acc);
                v = -acc / S[r][r];
            }
            y[r] = v;
            D[r * kCholNb + j] = v;
        }
    }
    for (int e = tid; e < kCholNb * kCholNb; e += 256) {
        const int r = e / kCholNb, c = e % kCholNb;
        if (r < nb && c <= r) A[(int64_t)(p + r) * K + p + c] = S[r][c];
    }
}

// Panel p, rows below the diagonal block: x = a L11^-T, i.e. x_c = sum_{s <= c} a_s D[c][s]
// (independent dot products; the thread owns its row segment, so it works in place).
__global__ void __launch_bounds__(128) chol_panel_kernel(double* __restrict__ A, int K, int p, int nb,
                                                         const double* __restrict__ Dinv)
{
    __shared__ double D[kCholNb][kCholNb + 1];
    const double* Dg = Dinv + (int64_t)(p / kCholNb) * kCholNb * kCholNb;
    for (int e = threadIdx.x; e < kCholNb * kCholNb; e += blockDim.x) D[e / kCholNb][e % kCholNb] = Dg[e];
    __syncthreads();
    const int r = p + nb + blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= K) return;
    double* row = A + (int64_t)r * K + p;
    double v[kCholNb];
#pragma unroll
    for (int s = 0; s < kCholNb; ++s) v[s] = s < nb ? row[s] : 0.0;
#pragma unroll 4
    for (int c = 0; c < nb; ++c) {
        double x = 0.0;
#pragma unroll
        for (int s = 0; s < kCholNb; ++s)
            if (s <= c) x = fma(v[s], D[c][s], x);
        row[c] = x;
    }
}

// Inverse, block row i (rows r0 .. r0+nb): on entry Linv[r0+r][j] (j < r0) holds
// T = L[i, <i] Linv[<i, <i]; it becomes -D_i T, and the diagonal block becomes D_i.
// One thread per column; the column's nb values are its own, so this works in place.
__global__ void __launch_bounds__(128) trinv_rows_kernel(double* __restrict__ Linv, int K, int r0, int nb,
                                                         const double* __restrict__ Dinv)
{
    __shared__ double D[kCholNb][kCholNb + 1];
    const double* Dg = Dinv + (int64_t)(r0 / kCholNb) * kCholNb * kCholNb;
    for (int e = threadIdx.x; e < kCholNb * kCholNb; e += blockDim.x) D[e / kCholNb][e % kCholNb] = Dg[e];
    __syncthreads();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= r0 + nb) return;
    double* col = Linv + (int64_t)r0 * K + j;
    if (j >= r0) {
        for (int r = 0; r < nb; ++r) col[(int64_t)r * K] = D[r][j - r0];
        return;
    }
    double y[kCholNb];
#pragma unroll
    for (int s = 0; s < kCholNb; ++s) y[s] = s < nb ? col[(int64_t)s * K] : 0.0;
#pragma unroll 4
    for (int r = 0; r < nb; ++r) {
        double x = 0.0;
#pragma unroll
        for (int s = 0; s < kCholNb; ++s)
            if (s <= r) x = fma(D[r][s], y[s], x);
        col[(int64_t)r * K] = -x;
    }
}

// One block of rows b .. b+B (one quantization group) for NC columns per CTA, 8 threads
// per column.  At the block's first row: the group's scale and zero from its compensated
// weights rounded to binary32 (range widened to contain 0, s = fp16 rounded up of r/15,
// z = round(-min/s) clamped to [0, 15]; a zero range gives 0 and 0).  Then row by row:
// the codes, err = (w - (q - z) s) / U[k][k] (kept in Err for the rows after the block)
// and w_j -= err U[k][j] for the later rows j of the block.
// U[k][j] = Linv[K-1-k][K-1-j].
__global__ void gptq_block_kernel(double* __restrict__ Wc, int K, int N, int b, int B,
                                  const double* __restrict__ Linv, uint8_t* __restrict__ codes,
                                  uint16_t* __restrict__ scales, uint8_t* __restrict__ zeros,
                                  double* __restrict__ Err, int NC)
{
    extern __shared__ double Ws[];  // [B][NC]
    const int c = threadIdx.x >> 3, sub = threadIdx.x & 7;
    const int n = blockIdx.x * NC + c;
    const bool live = n < N;
    for (int e = threadIdx.x; e < B * NC; e += blockDim.x) {
        const int r = e / NC, cc = e % NC, nn = blockIdx.x * NC + cc;
        Ws[e] = nn < N ? Wc[(int64_t)(b + r) * N + nn] : 0.0;
    }
    __syncthreads();
    // scale and zero (the 8 threads of a column share the scan)
    float mn = 0.0f, mx = 0.0f;
    for (int r = sub; r < B; r += 8) {
        const float v = __double2float_rn(Ws[r * NC + c]);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const float rng = __fsub_rn(mx, mn);
    const float s32 = __fdiv_rn(rng, 15.0f);
    __half s16 = __float2half_ru(s32);
    float s = __half2float(s16);
    int z = 0;
    if (rng == 0.0f) {
        s16 = __ushort_as_half((unsigned short)0);
        s = 0.0f;
    } else {
        z = min(max(__float2int_rn(__fdiv_rn(-mn, s)), 0), 15);
    }
    if (live && sub == 0) {
        if (s32 > 65504.0f) set_status(6u);
        const int g = b / B;
        scales[(int64_t)g * N + n] = __half_as_ushort(s16);
        zeros[(int64_t)g * N + n] = (uint8_t)z;
    }
    const double* Ub = Linv + (int64_t)(K - 1 - b) * K + (K - 1 - b);  // U[b+k][b+j] = Ub[-k K - j]
    for (int k = 0; k < B; ++k) {
        const double wd = Ws[k * NC + c];
        const float w = __double2float_rn(wd);
        const int q = s != 0.0f ? min(max(__float2int_rn(__fdiv_rn(w, s)) + z, 0), 15) : 0;
        const double err = (wd - (double)(q - z) * (double)s) / __ldg(Ub - (int64_t)k * K - k);
        if (live && sub == 0) {
            codes[(int64_t)(b + k) * N + n] = (uint8_t)q;
            Err[(int64_t)k * N + n] = err;
        }
        for (int j = k + 1 + sub; j < B; j += 8) Ws[j * NC + c] -= err * __ldg(Ub - (int64_t)k * K - j);
        __syncwarp();
    }
}

}  // namespace qg
