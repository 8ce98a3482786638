/*
 * qgemm.h -- C ABI of libqgemm.so, the B200 (sm_100a) quantized linear layer.
 *
 * What the library computes (the pages' definitions; page titles abbreviated):
 *   [Q]  "AI Infra guide, ch.4 Quantization" (aiinfra.vidrealm.tech), sec. 1.1-1.3:
 *        affine quantization x_int = round(x/s) + z, x_hat = (x_int - z) s;
 *        symmetric s = max|x|/127; asymmetric s = (max-min)/255 with z adjusted;
 *        per-channel / per-group / per-token granularity.
 *   [S]  same page, sec. 2.2 (SmoothQuant): Y = (X diag(s)^-1)(diag(s) W),
 *        s_j = max|X_j|^alpha / max|W_j|^(1-alpha), alpha = 0.5 typical.
 *   [W4] same page, sec. 3.1 and 3.5: weight-only INT4, dequantize and multiply,
 *        fused (Marlin-style) so that no dequantized copy of W is written.
 *   [G]  "LLM inference cost: W8A8/W4A8 ..." (0539edu.com), sec. 2.2: group-wise
 *        quantization with an independent scale and zero per group of 128; W4A8.
 *   [A]  "Quantization & Flash Attention -- LLM inference optimization (2)"
 *        (hustzhy.cn), sec. 2.1-2.3 (AWQ): per-input-channel scales
 *        s_c = mean(|X_c|)^alpha, X W = (X / s)(s W), alpha chosen on a grid in
 *        [0, 1] by the least MSE of the quantized layer's output.
 *
 * Readings taken where the pages are silent (the same ones the test oracle takes):
 *   asymmetric INT4 uses s = (max' - min')/15 over a range widened to contain 0,
 *   stored as fp16 rounded toward +infinity; z = clamp(round(-min'/s), 0, 15);
 *   code = clamp(round(x/s) + z, 0, 15) in that order; round = half to even in
 *   binary32; symmetric INT4 uses s = max|x|/7 (fp32) and codes in [-7, 7];
 *   INT8 codes lie in [-127, 127]; a zero range gives scale 0 and codes 0.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     keeps none of them after the call returns and allocates no device memory.
 *   - Tensors are dense and row-major: X[M][K] activations, W[K][N] weights,
 *     Y[M][N] = X W.  Groups run along K.
 *   - fp16 / bf16 tensors are passed as uint16_t bit patterns.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default stream).
 *     The return value reports argument validation and launch errors only; a
 *     call that returns anything but QG_OK launched nothing.
 *   - Conditions found on the device (a non-finite input, a scale that does not
 *     fit fp16, a bounded wait that ran out) set a sticky per-device status word
 *     instead; qg_device_status() synchronizes the stream, returns that word and
 *     clears it.
 *   - Shape rules common to all calls: M >= 0, K >= 1, N >= 1; M == 0 returns
 *     QG_OK and launches nothing.  Each call lists its own extra rules.
 *   - Base pointers must be 16-byte aligned (QG_ERR_ALIGN otherwise).
 */
#ifndef QGEMM_H
#define QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* qg_stream_t;

typedef enum {
    QG_OK = 0,
    QG_ERR_NULL = 1,        /* a required pointer is NULL */
    QG_ERR_SHAPE = 2,       /* a size breaks the call's shape rules */
    QG_ERR_ALIGN = 3,       /* a base pointer is not 16-byte aligned */
    QG_ERR_DTYPE = 4,       /* unknown dtype enumerator */
    QG_ERR_NONFINITE = 5,   /* (device) an input that must be finite was NaN or Inf */
    QG_ERR_RANGE = 6,       /* (device) a value outside its allowed range: an fp16 scale
                               that would overflow, an outlier offset outside its group,
                               a zero pivot in the GPTQ inverse */
    QG_ERR_TIMEOUT = 7,     /* (device) a bounded wait inside a kernel gave up */
    QG_ERR_CUDA = 8,        /* the CUDA runtime reported an error; see qg_last_error() */
    QG_ERR_UNSUPPORTED = 9, /* the device is not sm_100 or a feature is missing */
    QG_ERR_WORKSPACE = 10   /* workspace given but smaller than qg_workspace_size() */
} qg_status;

/* Operations that may use a caller-provided workspace (qg_workspace_size). */
typedef enum {
    QG_OP_GEMM_W4A16 = 0,
    QG_OP_GEMM_W8A8 = 1,
    QG_OP_GEMM_W4A8 = 2,
    QG_OP_AWQ_SEARCH = 3,
    QG_OP_GPTQ = 4
} qg_op;

typedef enum { QG_F16 = 0, QG_BF16 = 1 } qg_dtype;

/* --------------------------------------------------------------------------
 * Group-wise INT4 weight quantization.   [Q] sec. 1.1-1.3, [G] sec. 2.2
 *
 * W        fp32 [K][N].
 * s_smooth fp32 [K] or NULL.  When given, the quantized matrix is diag(s) W,
 *          i.e. W[k][n] * s_smooth[k] rounded once to fp32 ([S] sec. 2.2).
 * group    group size along K; K % group == 0, group % 8 == 0, 8 <= group <= 1024
 *          (128 everywhere in the workloads).
 * symmetric
 *   0: asymmetric.  codes u8 [K][N] in [0,15]; scales = fp16 bits [K/group][N]
 *      (uint16_t*), rounded toward +infinity; zeros u8 [K/group][N] in [0,15].
 *   1: symmetric.   codes = int8 [K][N] in [-7,7] (stored through the uint8_t*
 *      pointer as two's complement bytes); scales = fp32 [K/group][N]
 *      (float*); zeros must be NULL.
 * Device errors: QG_ERR_NONFINITE (a non-finite element; that group's outputs
 * are left unspecified), QG_ERR_RANGE (asymmetric scale above 65504).
 * ------------------------------------------------------------------------ */
qg_status qg_quantize_w4_group(const float* W, const float* s_smooth, int K, int N, int group,
                               int symmetric, uint8_t* codes, void* scales, uint8_t* zeros,
                               qg_stream_t stream);

/* --------------------------------------------------------------------------
 * Pack 4-bit codes 8 per uint32 along K, low nibble first:
 *   packed[kb][n] = sum_{i<8} (codes[8kb+i][n] & 0xF) << 4i
 * codes u8 [K][N] (symmetric codes as two's complement bytes), packed u32 [K/8][N].
 * K % 8 == 0.   (Storage of 8 nibbles per uint32, low first: [G] workload definition.)
 * ------------------------------------------------------------------------ */
qg_status qg_pack_nibbles(const uint8_t* codes, int K, int N, uint32_t* packed, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * W4A16 fused dequant-GEMM.   [W4] sec. 3.1, 3.5; [G] sec. 2.2 (pseudo-code of
 * the quantized matmul with per-group scale and zero)
 *
 *   Y[m][n] = sum_k X[m][k] * (q[k][n] - z[k/g][n]) * s[k/g][n]
 *
 * X        fp16 or bf16 [M][K] (xdt); Y has the same dtype, [M][N].
 * packed   u32 [K/8][N] from qg_pack_nibbles of asymmetric codes.
 * scales   fp16 bits [K/group][N]; zeros u8 [K/group][N].
 * group    128 (the only group size the GEMM kernels take).
 * Rules: K % 128 == 0, N % 8 == 0.  Accumulation is fp32.
 * workspace: NULL, or a device buffer of at least
 *   qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N) bytes; its contents on entry do
 *   not matter.  With a workspace, decode shapes (N % 16 == 0) use the stream-K
 *   kernel: the pieces of a column slab that is split between CTAs leave fp32
 *   partial tiles there, each published under a 64-bit token unique to the launch,
 *   and the CTA holding the slab's first piece adds them in a fixed order and
 *   writes Y (one launch per 32 tokens, deterministic).  Each launch leaves the
 *   tokens it consumed cleared.  The workspace must not be shared by calls that may
 *   run concurrently (calls in one stream are fine).  Without one, the split-K
 *   reduction runs in distributed shared memory (slower).
 *   The decode kernel starts streaming its weights, scales and zeros before the
 *   previous kernel in the stream has finished when that kernel allows it
 *   (programmatic dependent launch); X, Y and the workspace are touched only after
 *   it.  So packed, scales and zeros must not be written by a kernel that runs just
 *   before this call in the same stream and lets its dependents start early (no
 *   kernel of this library does).
 * ------------------------------------------------------------------------ */
qg_status qg_gemm_w4a16(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* packed,
                        const uint16_t* scales, const uint8_t* zeros, int group, void* Y,
                        void* workspace, size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * W4A16 GEMM that allocates nothing and takes no workspace.  The pages have no
 * counterpart to this call: it exists for callers that cannot allocate device
 * memory where they run the GEMM -- code inside a CUDA graph capture, operators
 * inside a framework that owns all device memory, latency-bound paths that cannot
 * afford an allocation's synchronisation.
 *
 * Same arguments and result as qg_gemm_w4a16 without (workspace, ws_bytes).  The
 * decode kernel's scratch lives in one static device array of 6 MiB per GPU
 * that loads the library, kept until the process exits; a shape whose scratch
 * would exceed it is refused with QG_ERR_WORKSPACE (see qg_last_error()).
 * The first call on each device looks the array's address up; make that first
 * call before any stream capture.  Nothing in the array needs to start at zero.
 * All calls share the one array: calls that may overlap on the GPU (other
 * streams, other threads) race and must not be issued.
 * ------------------------------------------------------------------------ */
qg_status qg_gemm_w4a16_noalloc(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* packed,
                                const uint16_t* scales, const uint8_t* zeros, int group, void* Y,
                                qg_stream_t stream);

/* --------------------------------------------------------------------------
 * Fused smoothing + per-token dynamic symmetric INT8 quantization of
 * activations.   [S] sec. 2.2; [Q] sec. 1.2 (s = max|x|/127), sec. 1.3 (per token)
 *
 *   X~[m][j] = X[m][j] * inv_s[j]           (one fp32 rounding; inv_s NULL -> X~ = X)
 *   t[m]     = max_j |X~[m][j]| / 127        (fp32)
 *   Xq[m][j] = clamp(round(X~[m][j] / t[m]), -127, 127);  t[m] == 0 -> all zero
 *
 * X bf16 [M][K]; inv_s fp32 [K] or NULL; Xq int8 [M][K]; t fp32 [M].
 * Rules: K % 8 == 0.   Device error: QG_ERR_NONFINITE.
 * ------------------------------------------------------------------------ */
qg_status qg_smooth_quant_act_i8(const uint16_t* X, int M, int K, const float* inv_s, int8_t* Xq,
                                 float* t, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * W8A8 GEMM (SmoothQuant).   [S] sec. 2.2-2.3; [Q] sec. 1.3
 *
 *   acc[m][n] = sum_k Xq[m][k] * Wq[k][n]          (int32, exact)
 *   Y[m][n]   = bf16_rn( ((float)acc * t[m]) * sw[n] )
 *
 * Xq int8 [M][K], t fp32 [M] (from qg_smooth_quant_act_i8); Wq int8 [K][N],
 * sw fp32 [N] (from qg_quantize_w8_channel); Y bf16 [M][N].
 * acc_dbg: NULL, or int32 [M][N] that also receives the exact accumulators.
 * Rules: K % 128 == 0, N % 16 == 0.
 * workspace: NULL, or (M < 128) a device buffer of at least
 *   qg_workspace_size(QG_OP_GEMM_W8A8, M, K, N) bytes (contents irrelevant: it holds
 *   per-launch 64-bit publication tokens and the int32 partial sums of column slabs
 *   split between CTAs, which the CTA holding a slab's first block adds in the same
 *   launch).  With it, M < 128 runs the stream-K tensor-core kernel (one launch); without
 *   it, the cluster split-K kernel.  Both give the same bits.  A workspace smaller than
 *   required -> QG_ERR_WORKSPACE before any launch.  Calls that may run concurrently need
 *   workspaces of their own.
 * ------------------------------------------------------------------------ */
qg_status qg_gemm_w8a8(const int8_t* Xq, const float* t, int M, int K, const int8_t* Wq,
                       const float* sw, int N, uint16_t* Y, int32_t* acc_dbg, void* workspace,
                       size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * W4A8 GEMM with per-group fp32 rescaling.   [G] sec. 2.2 (W4A8, group-wise)
 *
 *   P[m][g][n] = sum_{k in group g} Xq[m][k] * q[k][n]     (int32, exact)
 *   Y[m][n]    = bf16_rn( t[m] * sum_g P[m][g][n] * sg[g][n] )   (fp32)
 *
 * Xq int8 [M][K], t fp32 [M]; packed u32 [K/8][N] of symmetric codes (two's
 * complement nibbles in [-7,7]); sg fp32 [K/group][N]; Y bf16 [M][N].
 * part_dbg: NULL, or int32 [M][K/group][N] that also receives every P.
 * Rules: group == 128, K % 128 == 0, N % 16 == 0.
 * workspace: NULL, or (17 <= M < 128) a device buffer of at least
 *   qg_workspace_size(QG_OP_GEMM_W4A8, M, K, N) bytes (contents irrelevant: it holds
 *   per-launch publication tokens and the fp32 partial sums of column slabs split
 *   between CTAs, added in CTA order by the CTA holding a slab's first group in the same
 *   launch; the size is 0, and any workspace is ignored, for M <= 16 and M >= 128).
 *   With it, 17 <= M < 128 runs the stream-K tensor-core kernel (one launch per chunk)
 *   on chunks of up to 64 tokens; without it (and always at M <= 16), the cluster
 *   split-K kernel.  P is exact either way; Y may differ in the last bit (fp32 summation
 *   order).  A workspace smaller than required -> QG_ERR_WORKSPACE before any launch.
 *   Calls that may run concurrently need workspaces of their own.
 * ------------------------------------------------------------------------ */
qg_status qg_gemm_w4a8(const int8_t* Xq, const float* t, int M, int K, const uint32_t* packed,
                       const float* sg, int N, int group, uint16_t* Y, int32_t* part_dbg,
                       void* workspace, size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * SmoothQuant factors from a calibration batch.   [S] sec. 2.2
 *
 *   ax[j] = max_m |Xcal[m][j]|,  aw[j] = max_n |W[j][n]|
 *   s[j]  = ax^alpha / aw^(1-alpha)  (alpha == 0.5: sqrt(ax)/sqrt(aw) in fp32,
 *           correctly rounded; otherwise fp64 pow, rounded to fp32)
 *   s[j]  = 1 when ax or aw is 0;   inv_s[j] = 1 / s[j] (fp32)
 *
 * Xcal bf16 [Mc][K]; W fp32 [K][N]; s, inv_s fp32 [K].  0 <= alpha <= 1.
 * Device error: QG_ERR_NONFINITE.
 * ------------------------------------------------------------------------ */
qg_status qg_smooth_scales(const uint16_t* Xcal, int Mc, const float* W, int K, int N, float alpha,
                           float* s, float* inv_s, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * Per-output-channel symmetric INT8 weights.   [Q] sec. 1.2-1.3; [S] sec. 2.2
 *
 *   W~ = diag(s) W (s NULL -> W~ = W);  sw[n] = max_k |W~[k][n]| / 127
 *   Wq[k][n] = clamp(round(W~[k][n] / sw[n]), -127, 127);  sw[n] == 0 -> zeros
 *
 * W fp32 [K][N]; s fp32 [K] or NULL; Wq int8 [K][N]; sw fp32 [N].
 * Device error: QG_ERR_NONFINITE.
 * ------------------------------------------------------------------------ */
qg_status qg_quantize_w8_channel(const float* W, const float* s, int K, int N, int8_t* Wq, float* sw,
                                 qg_stream_t stream);

/* --------------------------------------------------------------------------
 * INT8 outlier side path beside the INT4 groups.   [G] sec. 2.2 (second technique)
 *
 * Split (offline), per group g of `group` rows along K and column n of
 * W~ = diag(s_smooth) W (or W):
 *   the `count` elements of largest |w| (ties: smaller k first), slot r = rank r:
 *     idx[g][r][n]    = their k offset inside the group (u8)
 *     s8[g][n]        = max |outlier| / 127 (fp32)
 *     codes8[g][r][n] = clamp(round(w / s8), -127, 127) (ties to even; s8 == 0 -> 0)
 *   W_dense = W~ with those elements set to 0 (fp32 [K][N]); it then goes through
 *   qg_quantize_w4_group (asymmetric) and qg_pack_nibbles as usual.
 * The pages keep the top 2% of each group: count = ceil(0.02 * group) = 3 for 128.
 * Rules: group % 8 == 0, 8 <= group <= 256, K % group == 0, 0 <= count <= 8
 * (count == 0: idx and codes8 may be NULL; s8 is set to 0 and W_dense = W~).
 * Device error: QG_ERR_NONFINITE (that group's outputs are then unspecified).
 * ------------------------------------------------------------------------ */
qg_status qg_outlier_split_w4(const float* W, const float* s_smooth, int K, int N, int group,
                              int count, uint8_t* idx, int8_t* codes8, float* s8, float* W_dense,
                              qg_stream_t stream);

/* Side path (run time): Y[m][n] = rn(Y[m][n] + sum_{g,r} X[m][g*group + idx] * codes8 * s8),
 * the sum in fp32 and one rounding back to the output dtype (= xdt, as for
 * qg_gemm_w4a16).  Same rules as the split; M == 0 or count == 0 launches nothing.
 * Device error: QG_ERR_RANGE when an idx entry is not below `group` (that entry is
 * skipped, never read past X). */
qg_status qg_outlier_side_add(const void* X, qg_dtype xdt, int M, int K, int N, int group,
                              int count, const uint8_t* idx, const int8_t* codes8,
                              const float* s8, void* Y, qg_stream_t stream);

/* The layer with the side path: Y = X deq4 + X deq8(outliers).
 * Fused (workspace given, at least qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N) bytes;
 *   1 <= count <= 4, group == 128, N % 16 == 0, and not bf16 with M >= 128): the decode
 *   kernel streams each group's offsets, codes and scales beside its INT4 words and adds
 *   the side sums (fp32, group then slot order) to the slab's fp32 sums, so Y is rounded
 *   once to the output dtype.  An offset not below the group sets QG_ERR_RANGE (skipped).
 * Otherwise: qg_gemm_w4a16 on the dense INT4 part, then qg_outlier_side_add (Y rounded
 *   twice).  Every argument is validated before anything launches. */
qg_status qg_gemm_w4a16_outlier(const void* X, qg_dtype xdt, int M, int K, int N,
                                const uint32_t* packed, const uint16_t* scales,
                                const uint8_t* zeros, int group, int count, const uint8_t* idx,
                                const int8_t* codes8, const float* s8, void* Y, void* workspace,
                                size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * 2:4 structured sparsity + INT4.   [G] sec. 3.2
 *
 * Prune: in every 4 consecutive rows k = 4b .. 4b+3 of a column the 2 elements of
 *   largest |w| are kept (ties: smaller k) and the other 2 set to 0 in Wp (fp32
 *   [K][N]); their positions i0 < i1 go to meta[b/8][n] as the nibble (i1 << 2) | i0
 *   at bits 4 (b mod 8) (u32 [K/32][N]).  Rules: K % 32 == 0.
 * Then: qg_quantize_w4_group(Wp, ..., symmetric = 0) as usual (the pruned zeros do
 *   not change a group's range), and the kept codes are packed with qg_pack24_vals:
 *   vals[kv/8][n] holds the kv-th kept code of column n (k order) at bits 4 (kv mod 8)
 *   (u32 [K/16][N]).  Rules: K % 32 == 0.
 * GEMM: Y = X * deq(W), pruned positions contributing exactly 0; fp32 accumulation,
 *   Y in the activation dtype.  Rules: group == 128, K % 128 == 0.  A SIMT kernel for
 *   few tokens (it reads 0.375 bytes per weight, positions included).
 * ------------------------------------------------------------------------ */
qg_status qg_prune24(const float* W, int K, int N, float* Wp, uint32_t* meta, qg_stream_t stream);
qg_status qg_pack24_vals(const uint8_t* codes, const uint32_t* meta, int K, int N, uint32_t* vals,
                         qg_stream_t stream);
qg_status qg_gemm_w4a16_24(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* vals,
                           const uint32_t* meta, const uint16_t* scales, const uint8_t* zeros,
                           int group, void* Y, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * Tensor-core form of the 2:4 GEMM (few tokens).   [G] sec. 3.2
 *
 * qg_pack24_tc: the kept codes of qg_pack24_vals rearranged for the sparse tensor-core
 *   instruction (mma.sp m16n8k32; an offline step, like packing): per group of 128 rows
 *   (32 blocks of 4) and column n, word vals_tc[8 gq + u][n], u = 2 t + hb (t = 0..3,
 *   hb = 0..1), holds for each 32-row step s = 0..3 of the group the two kept codes of
 *   block 8 s + t + 4 hb: the first (smaller k) at bits 4 s, the second at bits 16 + 4 s.
 *   vals u32 [K/16][N] (qg_pack24_vals) -> vals_tc u32 [K/16][N]; not in place.
 *   Rules: K % 128 == 0.
 * qg_gemm_w4a16_24_tc: Y = X * deq(W) as qg_gemm_w4a16_24 (pruned positions contribute
 *   exactly 0), from vals_tc, the position words meta (qg_prune24's, unchanged) and the
 *   asymmetric scales and zeros: a stream-K kernel streaming 0.375 byte per weight, each
 *   kept pair dequantized to (q - z) s in the activation dtype (exact subtraction, one
 *   rounding) and accumulated in fp32 by mma.sp.  Launches of up to 32 tokens.
 *   Rules: group == 128, K % 128 == 0, N % 32 == 0; workspace required, at least
 *   qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N) bytes (the decode kernel's contract:
 *   contents need no initialisation; concurrent calls must not share one).
 * ------------------------------------------------------------------------ */
qg_status qg_pack24_tc(const uint32_t* vals, int K, int N, uint32_t* vals_tc, qg_stream_t stream);
qg_status qg_gemm_w4a16_24_tc(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* vals_tc,
                              const uint32_t* meta, const uint16_t* scales, const uint8_t* zeros, int group,
                              void* Y, void* workspace, size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * GPTQ: INT4 weights with Hessian-weighted error compensation.   [A] sec. 3.1-3.3
 *
 *   H = (2/Mc) Xcal^T Xcal + lambda I, lambda = damp * trace / K (damp if the trace
 *   is 0), in binary64; H^-1 by Gauss-Jordan (no pivoting: H is positive definite).
 *   Rows k = 0 .. K-1 of W in order: at a group's first row the group's scale and
 *   zero (the asymmetric rules of qg_quantize_w4_group) from its compensated weights
 *   rounded to fp32; codes[k][n] = clamp(round(w / s) + z, 0, 15) on the compensated
 *   fp32 value; e = (w - (q - z) s) / H^-1[k][k]; w_j -= e H^-1[k][j] for j > k; then
 *   row and column k are eliminated from H^-1.  Every operation is one IEEE rounding
 *   in that order, so the results are reproducible bit for bit.
 * Xcal bf16 [Mc][K]; W fp32 [K][N]; codes u8 [K][N]; scales fp16 bits [K/group][N];
 * zeros u8 [K/group][N] (then qg_pack_nibbles and qg_gemm_w4a16 as usual).
 * Rules: Mc >= 1, 8 <= group <= 1024, group % 8 == 0, K % group == 0, K <= 16384,
 *   0 < damp (0.01 is the usual ridge).
 * workspace (required): at least qg_workspace_size(QG_OP_GPTQ, Mc, K, N) bytes
 *   (2 K^2 + K N doubles and a few vectors; more when the blocked form needs it),
 *   contents irrelevant.
 * Device errors: QG_ERR_NONFINITE (a non-finite weight), QG_ERR_RANGE (a scale above
 *   fp16, or a zero pivot).  An offline step: about 7 K kernel launches and
 *   O(K^3 + K^2 N) binary64 operations.
 * ------------------------------------------------------------------------ */
qg_status qg_gptq(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group,
                  double damp, uint8_t* codes, uint16_t* scales, uint8_t* zeros, void* workspace,
                  size_t ws_bytes, qg_stream_t stream);

/* GPTQ in its blocked Cholesky form (the fast offline path).   [A] sec. 3.1-3.3
 *
 *   Same H, lambda, group rules and outputs as qg_gptq.  After rows 0..k-1 are
 *   eliminated, row k of the remaining H^-1 over the square root of its diagonal is
 *   row k of the upper Cholesky factor U of H^-1 (H^-1 = U^T U), so with
 *   err_k = (w_k - (q_k - z) s) / U[k][k] and w_j -= err_k U[k][j] (j > k) each row is
 *   compensated as in qg_gptq.  U comes from one Cholesky factorization and one
 *   triangular inverse (U = J Lr^-1 J, Hr = J H J = Lr Lr^T, J the index reversal);
 *   the rows of a group are compensated inside the group as they are rounded and the
 *   later rows receive the group's errors in one GEMM per group.  All in binary64,
 *   summed in another order than qg_gptq: a code may differ from qg_gptq's where the
 *   compensated weight lies within rounding noise of a rounding boundary.
 * Arguments and rules as qg_gptq; workspace: qg_workspace_size(QG_OP_GPTQ, Mc, K, N)
 *   covers both forms.  Device errors: QG_ERR_NONFINITE (a non-finite weight),
 *   QG_ERR_RANGE (a scale above fp16, or a pivot that is not positive: H not positive
 *   definite in binary64).  About 6 K / 64 + 2 K / group kernel launches and
 *   O(K^3 / 3 + K^2 (Mc + N) / 2) binary64 multiply-adds.
 * ------------------------------------------------------------------------ */
qg_status qg_gptq_blocked(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group,
                          double damp, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                          void* workspace, size_t ws_bytes, qg_stream_t stream);

/* --------------------------------------------------------------------------
 * AWQ: activation-aware per-input-channel scales for the INT4 weights.   [A]
 *
 * Statistic (sec. 2.1):
 *   xm[c] = mean over the Mc calibration tokens of |Xcal[m][c]|: a binary64 sum
 *   over the tokens in order, divided by Mc in binary64, rounded once to fp32
 *   (the same bits on every run).
 * Xcal bf16 [Mc][K]; xm fp32 [K].  Rules: Mc >= 1, K >= 1.
 * ------------------------------------------------------------------------ */
qg_status qg_awq_act_mean(const uint16_t* Xcal, int Mc, int K, float* xm, qg_stream_t stream);

/* Scales for one exponent (sec. 2.3):
 *   s[c] = xm[c]^alpha (binary64 pow, rounded once to fp32); xm[c] == 0 -> s[c] = 1;
 *   inv_s[c] = 1 / s[c] (fp32, round to nearest).
 * Rules: K >= 1, 0 <= alpha <= 1. */
qg_status qg_awq_scales(const float* xm, int K, double alpha, float* s, float* inv_s,
                        qg_stream_t stream);

/* The scaled activations of the equivalent transform (sec. 2.2), in bf16:
 *   Xs[m][k] = bf16_rn(X[m][k] * inv_s[k])   (one fp32 product, one rounding)
 * X, Xs bf16 [M][K]; inv_s fp32 [K].  Rules: K % 8 == 0. */
qg_status qg_awq_scale_act(const uint16_t* X, int M, int K, const float* inv_s, uint16_t* Xs,
                           qg_stream_t stream);

/* The grid search (sec. 2.3), on the device, asynchronous on `stream`:
 *   alpha_i = i / (n_grid - 1), i = 0 .. n_grid-1 (alpha = 0 only when n_grid == 1);
 *   for each: s = xm^alpha; codes, scales, zeros = asymmetric INT4 groups of
 *   diag(s) W (qg_quantize_w4_group with s_smooth = s); Xs = qg_awq_scale_act(Xcal);
 *   Yq = qg_gemm_w4a16(Xs, ...) (bf16);
 *   mse[i] = mean over Mc x N of (Yref - Yq)^2 in binary64, where Yref = Xcal W
 *   with fp32 accumulation;
 *   best = the first i with the least mse[i]; s, inv_s = the scales at alpha_best.
 * Xcal bf16 [Mc][K]; W fp32 [K][N]; mse fp64 [n_grid]; best int32 [1]; s, inv_s
 * fp32 [K] (all device memory).  The winning weights are then
 * qg_quantize_w4_group(W, s, ...), and the layer's activations are scaled by inv_s
 * (qg_awq_scale_act, or folded into the producer of X).
 * Rules: group == 128, K % 128 == 0, N % 8 == 0, Mc >= 1, 1 <= n_grid <= 1024.
 * workspace (required): a device buffer of at least
 *   qg_workspace_size(QG_OP_AWQ_SEARCH, Mc, K, N) bytes, contents irrelevant.
 *   NULL -> QG_ERR_NULL; smaller -> QG_ERR_WORKSPACE, before any launch.
 * Device errors: those of the quantizer (QG_ERR_NONFINITE, QG_ERR_RANGE).
 * ------------------------------------------------------------------------ */
qg_status qg_awq_search(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group,
                        int n_grid, double* mse, int32_t* best, float* s, float* inv_s,
                        void* workspace, size_t ws_bytes, qg_stream_t stream);

/* Bytes of workspace the given operation and shape can use (0 = none).  The
 * value depends only on (op, M, K, N) and on the current device.  For
 * QG_OP_AWQ_SEARCH, M is the calibration token count Mc. */
size_t qg_workspace_size(qg_op op, int M, int K, int N);

/* --------------------------------------------------------------------------
 * Status and diagnostics
 * ------------------------------------------------------------------------ */

/* Synchronizes `stream`, returns the current device's sticky status word
 * (QG_OK if nothing was recorded) and clears it. */
qg_status qg_device_status(qg_stream_t stream);

/* Static, human-readable name of a status code. */
const char* qg_status_string(qg_status s);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* qg_last_error(void);

/* Test hook for the bounded-wait machinery: launches one block that waits on a
 * shared-memory barrier nothing will ever complete, giving up after `limit_ns`
 * nanoseconds (0 = the library default of 2 s).  The wait ends by itself; the
 * device status then reads QG_ERR_TIMEOUT.  No fault, trap or hang is involved. */
qg_status qg_selftest_bounded_wait(uint64_t limit_ns, qg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H */
