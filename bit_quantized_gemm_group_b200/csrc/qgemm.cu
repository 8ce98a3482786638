// qgemm.cu -- C ABI of libqgemm.so: argument validation, launch configuration and
// dispatch to the sm_100a kernels.  Declarations and full contracts: include/qgemm.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <type_traits>
#include <chrono>

#include "../../include/qgemm.h"
#include "act_quant.cuh"
#include "awq.cuh"
#include "gptq.cuh"
#include "gptq_blocked.cuh"
#include "common.cuh"
#include "int8_skinny.cuh"
#include "outlier.cuh"
#include "quantize.cuh"
#include "sparse24.cuh"
#include "tc_gemm.cuh"
#include "w4a16_decode.cuh"
#include "w4a16_tile.cuh"
#include "int8_decode.cuh"
#include "w4a8_decode.cuh"
#include "w4a16_skinny.cuh"

namespace {

thread_local char g_last_error[256] = "";

qg_status cuda_fail(cudaError_t e, const char* where)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return QG_ERR_CUDA;
}

#define QG_CUDA(call)                                      \
    do {                                                   \
        cudaError_t e_ = (call);                           \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
    } while (0)

bool misaligned(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u); }

// Per-device host caches (SM count, kernel occupancy, the no-alloc array's address)
// hold one slot per device index below kMaxDevices.  Slots are atomics: several host
// threads may make their first call on a device at once, and each then computes and
// stores the same value.  A device index beyond the slots is served without caching.
constexpr int kMaxDevices = 64;

// The calling thread's current device; QG_ERR_CUDA with the runtime's message when
// it cannot be determined.
qg_status current_device(int* dev)
{
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    return QG_OK;
}

bool cached_slot(int dev) { return dev >= 0 && dev < kMaxDevices; }

// SM count of the current device (148 on a B200).  Launch plans and workspace sizes
// are both derived from it, so a query failure here (reported again by the launch
// that follows) only changes the plan, never its consistency.
int num_sms()
{
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cached_slot(dev)) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (cached_slot(dev)) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Launch `kern` with a thread-block cluster of (1, cy, 1).
template <typename Kern, typename... Args>
qg_status launch_cluster(Kern kern, dim3 grid, dim3 block, size_t smem, int cy, qg_stream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = cy;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    QG_CUDA(cudaLaunchKernelEx(&cfg, kern, args...));
    return QG_OK;
}

// Choose the split-K cluster size S in {1,2,4,8} (S <= groups) that best fills the
// GPU: the fraction of CTA slots used over all waves, ties going to more CTAs.
int choose_split(int nslabs, int groups, int ctas_per_sm)
{
    const int slots = num_sms() * std::max(ctas_per_sm, 1);
    int best = 1;
    double best_eff = -1.0;
    for (int S = 1; S <= 8; S *= 2) {
        if (S > groups) break;
        const long total = (long)nslabs * S;
        const long waves = (total + slots - 1) / slots;
        const double eff = (double)total / (double)(waves * slots);
        if (eff > best_eff + 1e-9) {
            best_eff = eff;
            best = S;
        }
    }
    return best;
}

// Per kernel instance and device: raise the dynamic shared memory limit once and
// remember the occupancy, so that a launch makes no query calls after the first.  The
// occupancy is stored (release) only after the attribute is set, so a thread that
// reads it (acquire) launches with the attribute in place.
struct KernelInfo {
    std::atomic<int> occ[kMaxDevices];
};

template <typename Kern>
qg_status prepare_kernel(KernelInfo& info, Kern k, int threads, size_t smem, int* occ)
{
    int dev = 0;
    qg_status st = current_device(&dev);
    if (st != QG_OK) return st;
    if (cached_slot(dev)) {
        const int c = info.occ[dev].load(std::memory_order_acquire);
        if (c > 0) {
            *occ = c;
            return QG_OK;
        }
    }
    if (smem > 48 * 1024) QG_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    int n = 0;
    QG_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem));
    *occ = n > 0 ? n : 1;
    if (cached_slot(dev)) info.occ[dev].store(*occ, std::memory_order_release);
    return QG_OK;
}

// ---------------------------------------------------------------------------
// W4A16 skinny path (M <= 32 per launch)
// ---------------------------------------------------------------------------
template <int MT, bool BF16>
qg_status launch_w4a16_skinny(const qg::SkinnyParams& p, qg_stream_t stream)
{
    constexpr int WN = 2, WK = 4, DEPTH = 4;
    constexpr int BN = 64 * WN, MP = 8 * MT;
    auto kern = qg::w4a16_skinny_kernel<MT, BF16, WN, WK, DEPTH>;
    const size_t smem = (size_t)WK * BN * MP * 4;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, WN * WK * 32, smem, &occ);
    if (st != QG_OK) return st;
    const int nslabs = (p.N + BN - 1) / BN;
    const int S = choose_split(nslabs, p.K / 128, occ);
    return launch_cluster(kern, dim3(nslabs, S, 1), dim3(WN * WK * 32), smem, S, stream, p);
}

template <bool BF16>
qg_status w4a16_skinny_dispatch(qg::SkinnyParams p, qg_stream_t stream)
{
    for (int m0 = 0; m0 < p.M; m0 += 32) {
        qg::SkinnyParams q = p;
        q.M = std::min(32, p.M - m0);
        q.X = p.X + (int64_t)m0 * p.K;
        q.Y = p.Y + (int64_t)m0 * p.N;
        qg_status st;
        if (q.M <= 8) st = launch_w4a16_skinny<1, BF16>(q, stream);
        else if (q.M <= 16) st = launch_w4a16_skinny<2, BF16>(q, stream);
        else st = launch_w4a16_skinny<4, BF16>(q, stream);
        if (st != QG_OK) return st;
    }
    return QG_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime; no libcuda link)
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D tiled map over a row-major [outer][inner] array.
qg_status make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, size_t elem_bytes, const void* base, uint64_t inner,
                       uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw)
{
    auto enc = tmap_encoder();
    if (!enc) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
        return QG_ERR_UNSUPPORTED;
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * elem_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

// 3-D tiled map: dims {d0, d1, d2} with byte strides {stride1, stride2} for d1, d2.
qg_status make_tmap_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                       uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2,
                       CUtensorMapSwizzle sw)
{
    auto enc = tmap_encoder();
    if (!enc) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
        return QG_ERR_UNSUPPORTED;
    }
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

// N-D tiled map (rank 3..5): dims[0] is contiguous; strides[] are the byte strides of
// dims 1..rank-1, in any order.
qg_status make_tmap_nd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw)
{
    auto enc = tmap_encoder();
    if (!enc) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
        return QG_ERR_UNSUPPORTED;
    }
    cuuint64_t d[5], st[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
        if (i > 0) st[i - 1] = strides[i - 1];
    }
    CUresult r = enc(m, dt, rank, const_cast<void*>(base), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (%d-D) failed (%d)", rank, (int)r);
        return QG_ERR_CUDA;
    }
    return QG_OK;
}

// ---------------------------------------------------------------------------
// W4A16 decode (stream-K, TMA-fed, in-kernel finish of split slabs, workspace)
// ---------------------------------------------------------------------------
struct DecodePlan {
    int MP, G, nslabs, units, grid;
    size_t flags_bytes;    // [grid] u64 publication tokens, padded to 256 B
    size_t partial_bytes;  // flags + [grid] partial tiles of 128 x MP fp32
};

int decode_cps(int MP);  // CTAs per SM of the configuration for MP tokens (below)

// Launch plan of one decode launch of M <= 32 tokens.
DecodePlan decode_plan(int M, int K, int N)
{
    DecodePlan d;
    const int mc = std::min(M, 32);
    d.MP = mc <= 8 ? 8 : mc <= 16 ? 16 : 32;
    d.G = K / 128;
    d.nslabs = (N + qg::kDecBN - 1) / qg::kDecBN;
    d.units = d.G * d.nslabs;
    d.grid = std::min(decode_cps(d.MP) * num_sms(), d.units);
    d.flags_bytes = ((size_t)d.grid * 8 + 255) / 256 * 256;
    d.partial_bytes = d.flags_bytes + (size_t)d.grid * qg::kDecBN * d.MP * sizeof(float);
    return d;
}

// Workspace of a call: its launches (32 tokens each, then the remainder) run one after
// another in the stream and share it, so it covers the largest of their plans.
size_t decode_workspace_bytes(int M, int K, int N)
{
    size_t b = decode_plan(std::min(M, 32), K, N).partial_bytes;
    if (M > 32 && M % 32) b = std::max(b, decode_plan(M % 32, K, N).partial_bytes);
    return b;
}

bool decode_eligible(int M, int N) { return M >= 1 && N % 16 == 0; }

// Publication token of one decode launch: unique per launch within the process and
// never 0 (0 marks a consumed slot).  The sequence starts at a value drawn from the
// clock, so a workspace left over from another process (or any other contents)
// matches a live token only by a 2^-64 coincidence.
unsigned long long next_decode_token()
{
    static std::atomic<unsigned long long> ctr{0x9E3779B97F4A7C15ull ^
                                               (unsigned long long)std::chrono::steady_clock::now()
                                                   .time_since_epoch()
                                                   .count() *
                                                   0xBF58476D1CE4E5B9ull};
    unsigned long long t;
    do {
        t = ctr.fetch_add(1, std::memory_order_relaxed);
    } while (t == 0);
    return t;
}

template <typename Kern, typename... Args>
qg_status launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, qg_stream_t stream, Args... args)
{
    // programmatic dependent launch: the grid may start while the previous kernel in the
    // stream drains; the kernel orders itself with griddepcontrol.wait
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    QG_CUDA(cudaLaunchKernelEx(&cfg, kern, args...));
    return QG_OK;
}

// Launch configuration per token tile (MT n8 tiles of 8 tokens): consumer warps NW,
// groups per stage GPS, ring depth ST, dequantization mode FULL, producer warpgroup PWG
// (register split) or single producer warp, CTAs per SM of one launch CPS (the grid is
// CPS x the SM count) and the minimum resident CTAs per SM MINB the footprint is sized for
// (2: a CTA of the next call in the stream can be resident beside this one).
template <int MT> struct DecodeCfg;
template <> struct DecodeCfg<1> { static constexpr int NW = 8, GPS = 4, ST = 5, CPS = 1, MINB = 1; static constexpr bool FULL = false, PWG = true; };
template <> struct DecodeCfg<2> { static constexpr int NW = 8, GPS = 4, ST = 4, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
template <> struct DecodeCfg<4> { static constexpr int NW = 8, GPS = 2, ST = 4, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };

int decode_cps(int MP) { return MP <= 8 ? DecodeCfg<1>::CPS : MP <= 16 ? DecodeCfg<2>::CPS : DecodeCfg<4>::CPS; }

// 2:4 sparse INT4 (mma.sp): always the full dequantization; a group's weights take 6 KB
// of a stage instead of 8 KB, so the rings hold more groups.  CPS matches the dense
// configurations (one plan serves both).
template <int MT> struct DecodeCfgSp;
template <> struct DecodeCfgSp<1> { static constexpr int NW = 8, GPS = 4, ST = 6, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
template <> struct DecodeCfgSp<2> { static constexpr int NW = 8, GPS = 4, ST = 4, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
template <> struct DecodeCfgSp<4> { static constexpr int NW = 8, GPS = 2, ST = 5, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
// The outlier side path fused (OUT): each stage also holds the groups' outlier offsets,
// codes and scales (6 KB for 4 groups), so the rings are one stage shorter.
template <int MT> struct DecodeCfgOut;
template <> struct DecodeCfgOut<1> { static constexpr int NW = 8, GPS = 4, ST = 4, CPS = 1, MINB = 1; static constexpr bool FULL = false, PWG = true; };
template <> struct DecodeCfgOut<2> { static constexpr int NW = 8, GPS = 4, ST = 3, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
template <> struct DecodeCfgOut<4> { static constexpr int NW = 8, GPS = 2, ST = 3, CPS = 1, MINB = 1; static constexpr bool FULL = true, PWG = true; };
static_assert(DecodeCfgSp<1>::CPS == DecodeCfg<1>::CPS && DecodeCfgSp<2>::CPS == DecodeCfg<2>::CPS &&
                  DecodeCfgSp<4>::CPS == DecodeCfg<4>::CPS && DecodeCfgOut<1>::CPS == DecodeCfg<1>::CPS &&
                  DecodeCfgOut<2>::CPS == DecodeCfg<2>::CPS && DecodeCfgOut<4>::CPS == DecodeCfg<4>::CPS,
              "one decode plan for the dense, the 2:4 and the side-path kernels");

// The outlier side path of one decode launch (qg_gemm_w4a16_outlier's arrays).
struct DecodeOutliers {
    const uint8_t* idx;
    const int8_t* codes8;
    const float* s8;
    int count;
};

// SP: `packed` is the 2:4 kept-code array in the tensor-core layout (qg_pack24_tc) and
// `meta24` the position words; otherwise `packed` holds the dense words and meta24 is unused.
// OUT: the outlier side path `out` is fused (dense weights only).
template <int MT, bool BF16, bool SP = false, bool OUT = false>
qg_status launch_w4a16_decode(const qg::SkinnyParams& sp, const uint32_t* packed, const uint16_t* scales,
                              const uint8_t* zeros, void* ws, qg_stream_t stream, const uint32_t* meta24 = nullptr,
                              const DecodeOutliers* out = nullptr)
{
    using C = std::conditional_t<SP, DecodeCfgSp<MT>, std::conditional_t<OUT, DecodeCfgOut<MT>, DecodeCfg<MT>>>;
    using L = qg::DecodeSmem<MT, C::NW, C::GPS, C::ST, C::PWG, SP, OUT>;
    static_assert(C::MINB * (L::TOTAL + 1024) <= 228 * 1024, "decode kernel shared memory");
    auto kern = qg::w4a16_decode_kernel<MT, BF16, C::NW, C::GPS, C::ST, C::FULL, C::PWG, C::MINB, SP, OUT>;
    const size_t smem = L::TOTAL;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, L::THREADS, smem, &occ);
    if (st != QG_OK) return st;
    const DecodePlan d = decode_plan(sp.M, sp.K, sp.N);
    if (d.grid > C::CPS * num_sms()) return QG_ERR_UNSUPPORTED;  // plan and configuration disagree
    const bool narrow = sp.N % 32 != 0;
    if (SP && narrow) return QG_ERR_SHAPE;
    qg::DecodeMaps m;
    const uint64_t N = sp.N, K = sp.K, G = d.G;
    if (SP) {
        // kept codes {32 columns, 8 rows of a group, N/32 blocks, G groups}; position words
        // {32 columns, 4 rows of a group, N/32 blocks, G groups}; no swizzle (the lanes of a
        // warp read whole 128-byte rows)
        const uint64_t dv[4] = {32, 8, N / 32, G}, sv[3] = {N * 4, 128, 8 * N * 4};
        const uint64_t dm[4] = {32, 4, N / 32, G}, sm[3] = {N * 4, 128, 4 * N * 4};
        const uint32_t bvg[4] = {32, 8, 4, (uint32_t)C::GPS}, bv1[4] = {32, 8, 4, 1};
        const uint32_t bmg[4] = {32, 4, 4, (uint32_t)C::GPS}, bm1[4] = {32, 4, 4, 1};
        if ((st = make_tmap_nd(&m.wg, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, dv, sv, bvg,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
            (st = make_tmap_nd(&m.w1, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, dv, sv, bv1,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
            (st = make_tmap_nd(&m.mg, CU_TENSOR_MAP_DATA_TYPE_UINT32, meta24, 4, dm, sm, bmg,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
            (st = make_tmap_nd(&m.m1, CU_TENSOR_MAP_DATA_TYPE_UINT32, meta24, 4, dm, sm, bm1,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
            return st;
    } else if (narrow) {
        // [K/8][N] words, boxes {32 columns, 16 rows} (columns past N read as zero)
        if ((st = make_tmap_2d(&m.w1, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, N, K / 8, 32, 16,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
            return st;
        m.wg = m.w1;
    } else {
        // {32 columns, 16 rows of a group, N/32 column blocks, G groups}
        const uint64_t dims[4] = {32, 16, N / 32, G};
        const uint64_t strides[3] = {N * 4, 128, 16 * N * 4};
        const uint32_t boxg[4] = {32, 16, 4, (uint32_t)C::GPS};
        const uint32_t box1[4] = {32, 16, 4, 1};
        if ((st = make_tmap_nd(&m.wg, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, dims, strides, boxg,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK ||
            (st = make_tmap_nd(&m.w1, CU_TENSOR_MAP_DATA_TYPE_UINT32, packed, 4, dims, strides, box1,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
            return st;
    }
    // scales and zeros: {128 columns, GPS | 1 groups} (columns past N read as zero)
    if ((st = make_tmap_2d(&m.sg, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, scales, N, G, 128, C::GPS,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
        (st = make_tmap_2d(&m.s1, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, scales, N, G, 128, 1,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
        (st = make_tmap_2d(&m.zg, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, zeros, N, G, 128, C::GPS,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
        (st = make_tmap_2d(&m.z1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, zeros, N, G, 128, 1,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
        return st;
    // X as {64 k, M rows, K / 64 halves}: row stride K * 2 bytes, half stride 128 bytes
    if ((st = make_tmap_3d(&m.xg, CU_TENSOR_MAP_DATA_TYPE_UINT16, sp.X, 64, sp.M, K / 64, K * 2, 128, 64, 8 * MT,
                           2 * C::GPS, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK ||
        (st = make_tmap_3d(&m.x1, CU_TENSOR_MAP_DATA_TYPE_UINT16, sp.X, 64, sp.M, K / 64, K * 2, 128, 64, 8 * MT, 2,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
        return st;
    qg::DecodeParams p;
    p.ocount = 0;
    p.side_tx = 0;
    if (OUT) {
        if (!out || out->count < 1 || out->count > qg::kDecOutMax) return QG_ERR_SHAPE;
        const uint32_t cnt = (uint32_t)out->count;
        if ((st = make_tmap_3d(&m.oi, CU_TENSOR_MAP_DATA_TYPE_UINT8, out->idx, N, cnt, G, N, cnt * N, 128, cnt, C::GPS,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
            (st = make_tmap_3d(&m.oc, CU_TENSOR_MAP_DATA_TYPE_UINT8, out->codes8, N, cnt, G, N, cnt * N, 128, cnt,
                               C::GPS, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK ||
            (st = make_tmap_2d(&m.os, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, out->s8, N, G, 128, C::GPS,
                               CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
            return st;
        p.ocount = out->count;
        p.side_tx = (uint32_t)C::GPS * (2 * cnt * 128 + 512);
    }
    p.X = sp.X;
    p.scales = scales;
    p.zeros = zeros;
    p.Y = sp.Y;
    p.flags = static_cast<unsigned long long*>(ws);
    p.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + d.flags_bytes);
    p.token = next_decode_token();
    p.M = sp.M;
    p.K = sp.K;
    p.N = sp.N;
    p.G = d.G;
    p.nslabs = d.nslabs;
    p.units = d.units;
    p.grid = d.grid;
    p.narrow = narrow ? 1 : 0;
    return launch_pdl(kern, dim3(d.grid), dim3(L::THREADS), smem, stream, p, m);
}

template <bool BF16>
qg_status w4a16_decode_dispatch(qg::SkinnyParams p, const uint32_t* packed, const uint16_t* scales,
                                const uint8_t* zeros, void* ws, qg_stream_t stream)
{
    for (int m0 = 0; m0 < p.M; m0 += 32) {
        qg::SkinnyParams q = p;
        q.M = std::min(32, p.M - m0);
        q.X = p.X + (int64_t)m0 * p.K;
        q.Y = p.Y + (int64_t)m0 * p.N;
        qg_status st;
        if (q.M <= 8) st = launch_w4a16_decode<1, BF16>(q, packed, scales, zeros, ws, stream);
        else if (q.M <= 16) st = launch_w4a16_decode<2, BF16>(q, packed, scales, zeros, ws, stream);
        else st = launch_w4a16_decode<4, BF16>(q, packed, scales, zeros, ws, stream);
        if (st != QG_OK) return st;
    }
    return QG_OK;
}

// ---------------------------------------------------------------------------
// tcgen05 tile kernels (M >= kTcMinM)
// ---------------------------------------------------------------------------
template <int KIND>
qg_status launch_tc(const qg::TcParams& p, const CUtensorMap& ta, const CUtensorMap& tb, qg_stream_t stream)
{
    using C = qg::TcCfg<KIND>;
    auto kern = qg::tc_gemm_kernel<KIND>;
    const size_t smem = qg::TcSmem<KIND>::TOTAL;
    static_assert(qg::TcSmem<KIND>::TOTAL <= 227 * 1024, "tile kernel shared memory");
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, C::THREADS, smem, &occ);
    if (st != QG_OK) return st;
    const int tiles = p.m_tiles * p.n_tiles;
    const int grid = std::min(tiles, num_sms());
    kern<<<grid, C::THREADS, smem, reinterpret_cast<cudaStream_t>(stream)>>>(p, ta, tb);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status tc_w8a8(const qg::TcInt8Args& a, qg_stream_t stream)
{
    using C = qg::TcCfg<qg::TC_W8A8>;
    CUtensorMap ta, tb;
    qg_status st;
    if ((st = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    if ((st = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Wq, a.N, a.K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    qg::TcParams p{};
    p.t = a.t;
    p.sw = a.sw;
    p.Y = a.Y;
    p.dbg = a.dbg;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.m_tiles = (a.M + C::BM - 1) / C::BM;
    p.n_tiles = (a.N + C::BN - 1) / C::BN;
    return launch_tc<qg::TC_W8A8>(p, ta, tb, stream);
}

qg_status tc_w4a8(const qg::TcInt8Args& a, qg_stream_t stream)
{
    using C = qg::TcCfg<qg::TC_W4A8>;
    CUtensorMap ta, tb;
    qg_status st;
    if ((st = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    if ((st = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, a.N, a.K / 8, 128, 16,
                           CU_TENSOR_MAP_SWIZZLE_NONE)))
        return st;
    qg::TcParams p{};
    p.t = a.t;
    p.sg = a.sg;
    p.Y = a.Y;
    p.dbg = a.dbg;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.m_tiles = (a.M + C::BM - 1) / C::BM;
    p.n_tiles = (a.N + C::BN - 1) / C::BN;
    return launch_tc<qg::TC_W4A8>(p, ta, tb, stream);
}

qg_status tc_w4a16(const qg::TcW4A16Args& a, qg_stream_t stream)
{
    using C = qg::W4TileCfg;
    static_assert(C::TOTAL <= 227 * 1024, "W4A16 tile kernel shared memory");
    CUtensorMap tx, tw;
    qg_status st;
    if ((st = make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.X, a.K, a.M, C::BK, C::BT,
                           CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    if ((st = make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, a.N, a.K / 8, C::BW, C::BK / 8,
                           CU_TENSOR_MAP_SWIZZLE_NONE)))
        return st;
    qg::W4TileParams p{};
    p.scales = a.scales;
    p.zeros = a.zeros;
    p.Y = a.Y;
    p.M = a.M;
    p.K = a.K;
    p.N = a.N;
    p.t_tiles = (a.M + C::BT - 1) / C::BT;
    p.w_tiles = (a.N + C::BW - 1) / C::BW;
    auto kern = qg::w4a16_tile_kernel;
    static KernelInfo info;
    int occ = 1;
    if ((st = prepare_kernel(info, kern, C::THREADS, C::TOTAL, &occ)) != QG_OK) return st;
    const int grid = std::min(p.t_tiles * p.w_tiles, num_sms());
    kern<<<grid, C::THREADS, C::TOTAL, reinterpret_cast<cudaStream_t>(stream)>>>(p, tx, tw);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

// ---------------------------------------------------------------------------
// W8A8 decode (M < kTcMinM, stream-K on tcgen05, workspace)
// ---------------------------------------------------------------------------
struct I8Plan {
    int NT, KB, nslabs, units, grid;
    size_t flags_bytes;    // [grid] u64 publication tokens, padded to 256 B
    size_t partial_bytes;  // flags + [grid] published pieces of NT x 128 (4-byte elements)
};

I8Plan i8_plan(int M, int K, int N)
{
    I8Plan d;
    d.NT = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    d.KB = K / 128;
    d.nslabs = (N + 127) / 128;
    d.units = d.KB * d.nslabs;
    d.grid = std::min(std::min(num_sms(), d.units), 160);
    d.flags_bytes = ((size_t)d.grid * 8 + 255) / 256 * 256;
    d.partial_bytes = d.flags_bytes + (size_t)d.grid * 128 * d.NT * sizeof(int32_t);
    return d;
}

template <int NT>
qg_status launch_w8a8_decode(const int8_t* Xq, const float* t, int M, int K, const int8_t* Wq, const float* sw,
                             int N, uint16_t* Y, int32_t* acc_dbg, void* ws, qg_stream_t stream)
{
    using C = qg::I8DecCfg<NT>;
    static_assert(C::TOTAL <= 227 * 1024, "W8A8 decode kernel shared memory");
    auto kern = qg::w8a8_decode_kernel<NT>;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, C::THREADS, C::TOTAL, &occ);
    if (st != QG_OK) return st;
    const I8Plan d = i8_plan(M, K, N);
    CUtensorMap tw, tx;
    if ((st = make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Wq, N, K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) ||
        (st = make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Xq, K, M, 128, NT, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    qg::I8DecodeParams p{t,
                         sw,
                         Y,
                         acc_dbg,
                         reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + d.flags_bytes),
                         static_cast<unsigned long long*>(ws),
                         next_decode_token(),
                         M,
                         K,
                         N,
                         d.KB,
                         d.nslabs,
                         d.units,
                         d.grid};
    return launch_pdl(kern, dim3(d.grid), dim3(C::THREADS), C::TOTAL, stream, p, tw, tx);
}

// W4A8 stream-K (17 <= M < 128; M <= 64 per launch, larger M in chunks of 64 tokens).
// At 16 tokens and fewer the cluster split-K kernel is as fast or faster (measured at
// K = N = 8192: 16.4 vs 25.6 us at M = 1, 24.6 vs 25.6 us at M = 16).
constexpr int kW4A8DecodeMinM = 17;
constexpr int kW4A8DecodeMaxM = 64;
constexpr int kW4A8Issuers = 2;

I8Plan w4a8_plan(int M, int K, int N)
{
    I8Plan d;
    M = std::min(M, kW4A8DecodeMaxM);
    d.NT = M <= 32 ? 32 : 64;
    d.KB = K / 128;  // groups
    d.nslabs = (N + 127) / 128;
    d.units = d.KB * d.nslabs;
    d.grid = std::min(std::min(num_sms(), d.units), 160);
    d.flags_bytes = ((size_t)d.grid * 8 + 255) / 256 * 256;
    d.partial_bytes = d.flags_bytes + (size_t)d.grid * 128 * d.NT * sizeof(float);
    return d;
}

template <int NT>
qg_status launch_w4a8_decode(const int8_t* Xq, const float* t, int M, int K, const uint32_t* packed,
                             const float* sg, int N, uint16_t* Y, int32_t* part_dbg, void* ws, qg_stream_t stream)
{
    using C = qg::W4A8DecCfg<NT, kW4A8Issuers>;
    static_assert(C::TOTAL <= 227 * 1024, "W4A8 decode kernel shared memory");
    auto kern = qg::w4a8_decode_kernel<NT, kW4A8Issuers>;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, C::THREADS, C::TOTAL, &occ);
    if (st != QG_OK) return st;
    const I8Plan d = w4a8_plan(M, K, N);
    CUtensorMap tw, tx;
    if ((st = make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, N, K / 8, 128, 16,
                           CU_TENSOR_MAP_SWIZZLE_NONE)) ||
        (st = make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, Xq, K, M, 128, NT, CU_TENSOR_MAP_SWIZZLE_128B)))
        return st;
    qg::W4A8DecodeParams p{t,
                           sg,
                           Y,
                           part_dbg,
                           reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + d.flags_bytes),
                           static_cast<unsigned long long*>(ws),
                           next_decode_token(),
                           M,
                           K,
                           N,
                           d.KB,
                           d.nslabs,
                           d.units,
                           d.grid};
    return launch_pdl(kern, dim3(d.grid), dim3(C::THREADS), C::TOTAL, stream, p, tw, tx);
}

// AWQ search workspace: every buffer one candidate needs, 256-byte aligned pieces
struct AwqWs {
    float *xm, *sc, *inv;
    uint16_t* xs;
    uint8_t* codes;
    uint16_t* scales;
    uint8_t* zeros;
    uint32_t* packed;
    uint16_t* yq;
    float* yref;
    double* partials;
    size_t bytes;
};

AwqWs awq_carve(void* base, int Mc, int K, int N)
{
    AwqWs w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~size_t(255);
        return base ? static_cast<uint8_t*>(base) + o : nullptr;
    };
    const size_t G = (size_t)K / 128;
    w.xm = reinterpret_cast<float*>(take(4 * (size_t)K));
    w.sc = reinterpret_cast<float*>(take(4 * (size_t)K));
    w.inv = reinterpret_cast<float*>(take(4 * (size_t)K));
    w.xs = reinterpret_cast<uint16_t*>(take(2 * (size_t)Mc * K));
    w.codes = take((size_t)K * N);
    w.scales = reinterpret_cast<uint16_t*>(take(2 * G * N));
    w.zeros = take(G * N);
    w.packed = reinterpret_cast<uint32_t*>(take((size_t)K / 2 * N));
    w.yq = reinterpret_cast<uint16_t*>(take(2 * (size_t)Mc * N));
    w.yref = reinterpret_cast<float*>(take(4 * (size_t)Mc * N));
    w.partials = reinterpret_cast<double*>(take(8 * (size_t)qg::kAwqErrBlocks));
    w.bytes = off;
    return w;
}

// GPTQ workspace: the Gauss-Jordan matrix, the inverse Hessian, the pivot column, the
// compensated weights (binary64) and the per-column row state
struct GptqWs {
    double *a, *inv, *f, *wc, *e;
    float* s_col;
    int* z_col;
    size_t bytes;
};

GptqWs gptq_carve(void* base, int K, int N)
{
    GptqWs w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~size_t(255);
        return base ? static_cast<uint8_t*>(base) + o : nullptr;
    };
    w.a = reinterpret_cast<double*>(take(8 * (size_t)K * K));
    w.inv = reinterpret_cast<double*>(take(8 * (size_t)K * K));
    w.f = reinterpret_cast<double*>(take(8 * (size_t)K));
    w.wc = reinterpret_cast<double*>(take(8 * (size_t)K * N));
    w.e = reinterpret_cast<double*>(take(8 * (size_t)N));
    w.s_col = reinterpret_cast<float*>(take(4 * (size_t)N));
    w.z_col = reinterpret_cast<int*>(take(4 * (size_t)N));
    w.bytes = off;
    return w;
}

// Workspace of the blocked form: the reversed Hessian and its Cholesky factor (in
// place), the factor's inverse, the compensated weights, one block of row errors, the
// reversed calibration tokens and the inverses of the 64 x 64 diagonal blocks.
struct GptqBlockedWs {
    double *a, *inv, *wc, *err, *xr, *dinv;
    size_t bytes;
};

GptqBlockedWs gptq_blocked_carve(void* base, int Mc, int K, int N)
{
    GptqBlockedWs w{};
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~size_t(255);
        return base ? reinterpret_cast<double*>(static_cast<uint8_t*>(base) + o) : nullptr;
    };
    const size_t nblk = (size_t)(K + qg::kCholNb - 1) / qg::kCholNb;
    w.a = take(8 * (size_t)K * K);
    w.inv = take(8 * (size_t)K * K);
    w.wc = take(8 * (size_t)K * N);
    w.err = take(8 * (size_t)std::min(K, 1024) * N);
    w.xr = take(8 * (size_t)Mc * K);
    w.dinv = take(8 * nblk * qg::kCholNb * qg::kCholNb);
    w.bytes = off;
    return w;
}

template <int BM, int BN>
qg_status dgemm(const qg::DgemmArgs& a, cudaStream_t st)
{
    if (a.M <= 0 || a.N <= 0) return QG_OK;
    const dim3 grid((a.N + BN - 1) / BN, (a.M + BM - 1) / BM);
    qg::dgemm_strided_kernel<BM, BN><<<grid, 256, 0, st>>>(a);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

// ---------------------------------------------------------------------------
// int8 skinny paths
// ---------------------------------------------------------------------------
template <int MT>
qg_status launch_w8a8_skinny(const qg::Int8SkinnyParams& p, qg_stream_t stream)
{
    constexpr int WN = 1, WK = 8;
    constexpr int BN = 128 * WN, MP = 8 * MT;
    auto kern = qg::w8a8_skinny_kernel<MT, WN, WK>;
    const size_t smem = (size_t)WK * BN * MP * 4;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, WN * WK * 32, smem, &occ);
    if (st != QG_OK) return st;
    const int nslabs = (p.N + BN - 1) / BN;
    const int S = choose_split(nslabs, p.K / 128, occ);
    return launch_cluster(kern, dim3(nslabs, S, 1), dim3(WN * WK * 32), smem, S, stream, p);
}

template <int MT>
qg_status launch_w4a8_skinny(const qg::Int8SkinnyParams& p, qg_stream_t stream)
{
    constexpr int WN = 2, WK = 4;
    constexpr int BN = 64 * WN, MP = 8 * MT;
    auto kern = qg::w4a8_skinny_kernel<MT, WN, WK>;
    const size_t smem = (size_t)WK * BN * MP * 4;
    static KernelInfo info;
    int occ = 1;
    qg_status st = prepare_kernel(info, kern, WN * WK * 32, smem, &occ);
    if (st != QG_OK) return st;
    const int nslabs = (p.N + BN - 1) / BN;
    const int S = choose_split(nslabs, p.K / 128, occ);
    return launch_cluster(kern, dim3(nslabs, S, 1), dim3(WN * WK * 32), smem, S, stream, p);
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* qg_status_string(qg_status s)
{
    switch (s) {
        case QG_OK: return "QG_OK";
        case QG_ERR_NULL: return "QG_ERR_NULL";
        case QG_ERR_SHAPE: return "QG_ERR_SHAPE";
        case QG_ERR_ALIGN: return "QG_ERR_ALIGN";
        case QG_ERR_DTYPE: return "QG_ERR_DTYPE";
        case QG_ERR_NONFINITE: return "QG_ERR_NONFINITE";
        case QG_ERR_RANGE: return "QG_ERR_RANGE";
        case QG_ERR_TIMEOUT: return "QG_ERR_TIMEOUT";
        case QG_ERR_CUDA: return "QG_ERR_CUDA";
        case QG_ERR_UNSUPPORTED: return "QG_ERR_UNSUPPORTED";
        case QG_ERR_WORKSPACE: return "QG_ERR_WORKSPACE";
    }
    return "QG_ERR_UNKNOWN";
}

const char* qg_last_error(void) { return g_last_error; }

size_t qg_workspace_size(qg_op op, int M, int K, int N)
{
    if (op == QG_OP_GPTQ) {  // any K that a group size divides (K % 8 == 0), any N
        if (M < 1 || K < 8 || K % 8 || K > 16384 || N < 1) return 0;
        return std::max(gptq_carve(nullptr, K, N).bytes, gptq_blocked_carve(nullptr, M, K, N).bytes);
    }
    if (M < 1 || K < 128 || N < 8 || K % 128) return 0;
    switch (op) {
        case QG_OP_GEMM_W4A16: {
            if (!decode_eligible(M, N)) return 0;
            return decode_workspace_bytes(M, K, N);
        }
        case QG_OP_GEMM_W8A8: {
            if (M >= qg::kTcMinM || N % 16) return 0;
            return i8_plan(M, K, N).partial_bytes;
        }
        case QG_OP_AWQ_SEARCH: {
            if (N % 8) return 0;
            return awq_carve(nullptr, M, K, N).bytes;
        }
        case QG_OP_GEMM_W4A8: {
            if (M < kW4A8DecodeMinM || M >= qg::kTcMinMW4A8 || N % 16) return 0;
            return w4a8_plan(M, K, N).partial_bytes;
        }
        default: return 0;
    }
}

qg_status qg_device_status(qg_stream_t stream)
{
    QG_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    unsigned int v = 0, zero = 0;
    QG_CUDA(cudaMemcpyFromSymbol(&v, qg::g_status, sizeof(v)));
    QG_CUDA(cudaMemcpyToSymbol(qg::g_status, &zero, sizeof(zero)));
    return (qg_status)v;
}

qg_status qg_quantize_w4_group(const float* W, const float* s_smooth, int K, int N, int group, int symmetric,
                               uint8_t* codes, void* scales, uint8_t* zeros, qg_stream_t stream)
{
    if (!W || !codes || !scales || (!symmetric && !zeros)) return QG_ERR_NULL;
    if (symmetric && zeros) return QG_ERR_NULL;
    if (K < 1 || N < 1 || group < 8 || group > 1024 || group % 8 || K % group) return QG_ERR_SHAPE;
    if (misaligned(W) || misaligned(s_smooth) || misaligned(codes) || misaligned(scales) || misaligned(zeros))
        return QG_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((group == 64 || group == 128 || group == 256) && N % 4 == 0) {
        // one pass over W with 16-byte accesses, values held in registers
        const dim3 g4((N + 127) / 128, K / group), b4(512);
        uint16_t* sc16 = static_cast<uint16_t*>(scales);
        if (group == 64)
            symmetric ? qg::quantize_w4_vec_kernel<64, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_vec_kernel<64, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        else if (group == 128)
            symmetric ? qg::quantize_w4_vec_kernel<128, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_vec_kernel<128, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        else
            symmetric ? qg::quantize_w4_vec_kernel<256, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_vec_kernel<256, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        QG_CUDA(cudaGetLastError());
        return QG_OK;
    }
    if (group == 64 || group == 128 || group == 256) {
        // one pass over W, values held in registers
        const dim3 g4((N + 127) / 128, K / group), b4(512);
        uint16_t* sc16 = static_cast<uint16_t*>(scales);
        if (group == 64)
            symmetric ? qg::quantize_w4_regs_kernel<64, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_regs_kernel<64, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        else if (group == 128)
            symmetric ? qg::quantize_w4_regs_kernel<128, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_regs_kernel<128, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        else
            symmetric ? qg::quantize_w4_regs_kernel<256, true><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, scales, nullptr)
                      : qg::quantize_w4_regs_kernel<256, false><<<g4, b4, 0, s>>>(W, s_smooth, K, N, codes, sc16, zeros);
        QG_CUDA(cudaGetLastError());
        return QG_OK;
    }
    const dim3 grid((N + 255) / 256, K / group), block(256);
    if (symmetric)
        qg::quantize_w4_sym_kernel<<<grid, block, 0, s>>>(W, s_smooth, K, N, group, reinterpret_cast<int8_t*>(codes),
                                                           static_cast<float*>(scales));
    else
        qg::quantize_w4_asym_kernel<<<grid, block, 0, s>>>(W, s_smooth, K, N, group, codes,
                                                            static_cast<uint16_t*>(scales), zeros);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_pack_nibbles(const uint8_t* codes, int K, int N, uint32_t* packed, qg_stream_t stream)
{
    if (!codes || !packed) return QG_ERR_NULL;
    if (K < 8 || N < 1 || K % 8) return QG_ERR_SHAPE;
    if (misaligned(codes) || misaligned(packed)) return QG_ERR_ALIGN;
    const dim3 grid(((N + 3) / 4 + 255) / 256, K / 8), block(256);
    qg::pack_nibbles_kernel<<<grid, block, 0, reinterpret_cast<cudaStream_t>(stream)>>>(codes, K, N, packed);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_gemm_w4a16(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* packed,
                        const uint16_t* scales, const uint8_t* zeros, int group, void* Y, void* workspace,
                        size_t ws_bytes, qg_stream_t stream)
{
    if (xdt != QG_F16 && xdt != QG_BF16) return QG_ERR_DTYPE;
    if (M < 0 || K < 128 || N < 8 || K % 128 || N % 8 || group != 128) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!X || !packed || !scales || !zeros || !Y) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(packed) || misaligned(scales) || misaligned(zeros) || misaligned(Y))
        return QG_ERR_ALIGN;
    if (xdt == QG_BF16 && M >= qg::kTcMinM) {
        qg::TcW4A16Args a{static_cast<const uint16_t*>(X), packed, scales, zeros, static_cast<uint16_t*>(Y), M, K, N};
        return tc_w4a16(a, stream);
    }
    qg::SkinnyParams p{static_cast<const uint16_t*>(X), packed, scales, zeros, static_cast<uint16_t*>(Y), M, K, N};
    if (workspace && decode_eligible(M, N)) {
        if (ws_bytes < qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N)) return QG_ERR_WORKSPACE;
        if (misaligned(workspace)) return QG_ERR_ALIGN;
        return xdt == QG_BF16 ? w4a16_decode_dispatch<true>(p, packed, scales, zeros, workspace, stream)
                              : w4a16_decode_dispatch<false>(p, packed, scales, zeros, workspace, stream);
    }
    return xdt == QG_BF16 ? w4a16_skinny_dispatch<true>(p, stream) : w4a16_skinny_dispatch<false>(p, stream);
}

qg_status qg_smooth_quant_act_i8(const uint16_t* X, int M, int K, const float* inv_s, int8_t* Xq, float* t,
                                 qg_stream_t stream)
{
    if (M < 0 || K < 8 || K % 8) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!X || !Xq || !t) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(inv_s) || misaligned(Xq) || misaligned(t)) return QG_ERR_ALIGN;
    qg::smooth_quant_act_i8_kernel<<<M, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(X, K, inv_s, Xq, t);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_gemm_w8a8(const int8_t* Xq, const float* t, int M, int K, const int8_t* Wq, const float* sw, int N,
                       uint16_t* Y, int32_t* acc_dbg, void* workspace, size_t ws_bytes, qg_stream_t stream)
{
    if (M < 0 || K < 128 || N < 16 || K % 128 || N % 16) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!Xq || !t || !Wq || !sw || !Y) return QG_ERR_NULL;
    if (misaligned(Xq) || misaligned(t) || misaligned(Wq) || misaligned(sw) || misaligned(Y) || misaligned(acc_dbg) ||
        misaligned(workspace))
        return QG_ERR_ALIGN;
    if (M >= qg::kTcMinM) {
        qg::TcInt8Args a{Xq, t, Wq, sw, nullptr, nullptr, Y, acc_dbg, M, K, N};
        return tc_w8a8(a, stream);
    }
    if (workspace) {
        if (ws_bytes < qg_workspace_size(QG_OP_GEMM_W8A8, M, K, N)) return QG_ERR_WORKSPACE;
        const int nt = i8_plan(M, K, N).NT;
        return nt == 16   ? launch_w8a8_decode<16>(Xq, t, M, K, Wq, sw, N, Y, acc_dbg, workspace, stream)
               : nt == 32 ? launch_w8a8_decode<32>(Xq, t, M, K, Wq, sw, N, Y, acc_dbg, workspace, stream)
               : nt == 64 ? launch_w8a8_decode<64>(Xq, t, M, K, Wq, sw, N, Y, acc_dbg, workspace, stream)
                          : launch_w8a8_decode<128>(Xq, t, M, K, Wq, sw, N, Y, acc_dbg, workspace, stream);
    }
    for (int m0 = 0; m0 < M; m0 += 16) {
        qg::Int8SkinnyParams p{Xq + (int64_t)m0 * K, t + m0, Wq, sw, nullptr, nullptr, Y + (int64_t)m0 * N,
                               acc_dbg ? acc_dbg + (int64_t)m0 * N : nullptr, std::min(16, M - m0), K, N};
        qg_status st = p.M <= 8 ? launch_w8a8_skinny<1>(p, stream) : launch_w8a8_skinny<2>(p, stream);
        if (st != QG_OK) return st;
    }
    return QG_OK;
}

qg_status qg_gemm_w4a8(const int8_t* Xq, const float* t, int M, int K, const uint32_t* packed, const float* sg,
                       int N, int group, uint16_t* Y, int32_t* part_dbg, void* workspace, size_t ws_bytes,
                       qg_stream_t stream)
{
    if (M < 0 || K < 128 || N < 16 || K % 128 || N % 16 || group != 128) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!Xq || !t || !packed || !sg || !Y) return QG_ERR_NULL;
    if (misaligned(Xq) || misaligned(t) || misaligned(packed) || misaligned(sg) || misaligned(Y) ||
        misaligned(part_dbg) || misaligned(workspace))
        return QG_ERR_ALIGN;
    if (M >= qg::kTcMinMW4A8) {
        qg::TcInt8Args a{Xq, t, nullptr, nullptr, packed, sg, Y, part_dbg, M, K, N};
        return tc_w4a8(a, stream);
    }
    const int G = K / 128;
    if (workspace && M >= kW4A8DecodeMinM) {
        if (ws_bytes < qg_workspace_size(QG_OP_GEMM_W4A8, M, K, N)) return QG_ERR_WORKSPACE;
        for (int m0 = 0; m0 < M; m0 += kW4A8DecodeMaxM) {
            // chunks run in stream order; each reuses the workspace after the previous chunk's launch
            // (a ragged last chunk of 16 tokens or fewer runs on the 32-token tile)
            const int mc = std::min(kW4A8DecodeMaxM, M - m0);
            const int nt = w4a8_plan(mc, K, N).NT;
            const int8_t* xc = Xq + (int64_t)m0 * K;
            uint16_t* yc = Y + (int64_t)m0 * N;
            int32_t* dc = part_dbg ? part_dbg + (int64_t)m0 * G * N : nullptr;
            qg_status st = nt == 32 ? launch_w4a8_decode<32>(xc, t + m0, mc, K, packed, sg, N, yc, dc, workspace, stream)
                                    : launch_w4a8_decode<64>(xc, t + m0, mc, K, packed, sg, N, yc, dc, workspace, stream);
            if (st != QG_OK) return st;
        }
        return QG_OK;
    }
    for (int m0 = 0; m0 < M; m0 += 32) {
        qg::Int8SkinnyParams p{Xq + (int64_t)m0 * K, t + m0, nullptr, nullptr, packed, sg, Y + (int64_t)m0 * N,
                               part_dbg ? part_dbg + (int64_t)m0 * G * N : nullptr, std::min(32, M - m0), K, N};
        qg_status st = p.M <= 8 ? launch_w4a8_skinny<1>(p, stream)
                       : p.M <= 16 ? launch_w4a8_skinny<2>(p, stream)
                                   : launch_w4a8_skinny<4>(p, stream);
        if (st != QG_OK) return st;
    }
    return QG_OK;
}

qg_status qg_smooth_scales(const uint16_t* Xcal, int Mc, const float* W, int K, int N, float alpha, float* s,
                           float* inv_s, qg_stream_t stream)
{
    if (!Xcal || !W || !s || !inv_s) return QG_ERR_NULL;
    if (Mc < 1 || K < 1 || N < 1) return QG_ERR_SHAPE;
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return QG_ERR_SHAPE;
    if (misaligned(Xcal) || misaligned(W) || misaligned(s) || misaligned(inv_s)) return QG_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    qg::col_absmax_bf16_kernel<<<(K + 255) / 256, 256, 0, st>>>(Xcal, Mc, K, s);
    QG_CUDA(cudaGetLastError());
    qg::row_absmax_f32_kernel<<<K, 256, 0, st>>>(W, K, N, inv_s);
    QG_CUDA(cudaGetLastError());
    qg::smooth_finalize_kernel<<<(K + 255) / 256, 256, 0, st>>>(s, inv_s, K, alpha);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_outlier_split_w4(const float* W, const float* s_smooth, int K, int N, int group, int count,
                              uint8_t* idx, int8_t* codes8, float* s8, float* W_dense, qg_stream_t stream)
{
    if (!W || !s8 || !W_dense || (count > 0 && (!idx || !codes8))) return QG_ERR_NULL;
    if (K < 1 || N < 1 || group < 8 || group > 256 || group % 8 || K % group || count < 0 ||
        count > qg::kMaxOutliers || count > group)
        return QG_ERR_SHAPE;
    if (misaligned(W) || misaligned(s_smooth) || misaligned(idx) || misaligned(codes8) || misaligned(s8) ||
        misaligned(W_dense))
        return QG_ERR_ALIGN;
    const dim3 grid((N + 255) / 256, K / group), block(256);
    qg::outlier_split_kernel<<<grid, block, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, s_smooth, K, N, group, count,
                                                                                          idx, codes8, s8, W_dense);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

namespace {
qg_status outlier_side_args(const void* X, qg_dtype xdt, int M, int K, int N, int group, int count,
                            const uint8_t* idx, const int8_t* codes8, const float* s8, const void* Y)
{
    if (xdt != QG_F16 && xdt != QG_BF16) return QG_ERR_DTYPE;
    if (M < 0 || K < 1 || N < 1 || group < 8 || group > 256 || group % 8 || K % group || count < 0 ||
        count > qg::kMaxOutliers || count > group)
        return QG_ERR_SHAPE;
    if (M > 0 && count > 0 && (!X || !idx || !codes8 || !s8 || !Y)) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(idx) || misaligned(codes8) || misaligned(s8) || misaligned(Y)) return QG_ERR_ALIGN;
    return QG_OK;
}

qg_status outlier_side_launch(const void* X, qg_dtype xdt, int M, int K, int N, int group, int count,
                              const uint8_t* idx, const int8_t* codes8, const float* s8, void* Y, qg_stream_t stream)
{
    if (M == 0 || count == 0) return QG_OK;
    constexpr int MT = 8;
    const dim3 grid((N + 127) / 128, (M + MT - 1) / MT), block(128);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (xdt == QG_BF16)
        qg::outlier_side_add_kernel<MT, true><<<grid, block, 0, st>>>(x, M, K, N, group, count, idx, codes8, s8, y);
    else
        qg::outlier_side_add_kernel<MT, false><<<grid, block, 0, st>>>(x, M, K, N, group, count, idx, codes8, s8, y);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}
}  // namespace

qg_status qg_outlier_side_add(const void* X, qg_dtype xdt, int M, int K, int N, int group, int count,
                              const uint8_t* idx, const int8_t* codes8, const float* s8, void* Y, qg_stream_t stream)
{
    qg_status st = outlier_side_args(X, xdt, M, K, N, group, count, idx, codes8, s8, Y);
    if (st != QG_OK) return st;
    return outlier_side_launch(X, xdt, M, K, N, group, count, idx, codes8, s8, Y, stream);
}

qg_status qg_gemm_w4a16_outlier(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* packed,
                                const uint16_t* scales, const uint8_t* zeros, int group, int count,
                                const uint8_t* idx, const int8_t* codes8, const float* s8, void* Y, void* workspace,
                                size_t ws_bytes, qg_stream_t stream)
{
    qg_status st = outlier_side_args(X, xdt, M, K, N, group, count, idx, codes8, s8, Y);
    if (st != QG_OK) return st;
    if (M == 0) return QG_OK;
    if (workspace && count >= 1 && count <= qg::kDecOutMax && group == 128 && K >= 128 && K % 128 == 0 &&
        decode_eligible(M, N) && !(xdt == QG_BF16 && M >= qg::kTcMinM)) {
        // the side path fused into the decode kernel: Y rounded once
        if (!packed || !scales || !zeros) return QG_ERR_NULL;
        if (misaligned(packed) || misaligned(scales) || misaligned(zeros) || misaligned(workspace)) return QG_ERR_ALIGN;
        if (ws_bytes < qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N)) return QG_ERR_WORKSPACE;
        const DecodeOutliers o{idx, codes8, s8, count};
        const uint16_t* x = static_cast<const uint16_t*>(X);
        uint16_t* y = static_cast<uint16_t*>(Y);
        for (int m0 = 0; m0 < M; m0 += 32) {
            qg::SkinnyParams q{x + (int64_t)m0 * K, packed, scales, zeros, y + (int64_t)m0 * N, std::min(32, M - m0), K, N};
            if (xdt == QG_BF16) {
                if (q.M <= 8) st = launch_w4a16_decode<1, true, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
                else if (q.M <= 16) st = launch_w4a16_decode<2, true, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
                else st = launch_w4a16_decode<4, true, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
            } else {
                if (q.M <= 8) st = launch_w4a16_decode<1, false, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
                else if (q.M <= 16) st = launch_w4a16_decode<2, false, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
                else st = launch_w4a16_decode<4, false, false, true>(q, packed, scales, zeros, workspace, stream, nullptr, &o);
            }
            if (st != QG_OK) return st;
        }
        return QG_OK;
    }
    if ((st = qg_gemm_w4a16(X, xdt, M, K, N, packed, scales, zeros, group, Y, workspace, ws_bytes, stream)) != QG_OK)
        return st;
    return outlier_side_launch(X, xdt, M, K, N, group, count, idx, codes8, s8, Y, stream);
}

qg_status qg_prune24(const float* W, int K, int N, float* Wp, uint32_t* meta, qg_stream_t stream)
{
    if (!W || !Wp || !meta) return QG_ERR_NULL;
    if (K < 32 || K % 32 || N < 1) return QG_ERR_SHAPE;
    if (misaligned(W) || misaligned(Wp) || misaligned(meta)) return QG_ERR_ALIGN;
    qg::prune24_kernel<<<dim3((N + 255) / 256, K / 32), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, K, N, Wp,
                                                                                                          meta);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_pack24_vals(const uint8_t* codes, const uint32_t* meta, int K, int N, uint32_t* vals, qg_stream_t stream)
{
    if (!codes || !meta || !vals) return QG_ERR_NULL;
    if (K < 32 || K % 32 || N < 1) return QG_ERR_SHAPE;
    if (misaligned(codes) || misaligned(meta) || misaligned(vals)) return QG_ERR_ALIGN;
    qg::pack24_kernel<<<dim3((N + 255) / 256, K / 16), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(codes, meta, K,
                                                                                                         N, vals);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_gemm_w4a16_24(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* vals,
                           const uint32_t* meta, const uint16_t* scales, const uint8_t* zeros, int group, void* Y,
                           qg_stream_t stream)
{
    if (xdt != QG_F16 && xdt != QG_BF16) return QG_ERR_DTYPE;
    if (M < 0 || K < 128 || K % 128 || N < 1 || group != 128) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!X || !vals || !meta || !scales || !zeros || !Y) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(vals) || misaligned(meta) || misaligned(scales) || misaligned(zeros) ||
        misaligned(Y))
        return QG_ERR_ALIGN;
    constexpr int MT = 8;
    const dim3 grid((N + 127) / 128, (M + MT - 1) / MT), block(128);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    if (xdt == QG_BF16)
        qg::gemm_w4a16_24_kernel<MT, true><<<grid, block, 0, st>>>(x, M, K, N, vals, meta, scales, zeros, y);
    else
        qg::gemm_w4a16_24_kernel<MT, false><<<grid, block, 0, st>>>(x, M, K, N, vals, meta, scales, zeros, y);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_pack24_tc(const uint32_t* vals, int K, int N, uint32_t* vals_tc, qg_stream_t stream)
{
    if (!vals || !vals_tc) return QG_ERR_NULL;
    if (K < 128 || K % 128 || N < 1) return QG_ERR_SHAPE;
    if (misaligned(vals) || misaligned(vals_tc)) return QG_ERR_ALIGN;
    if (vals == vals_tc) return QG_ERR_SHAPE;  // not in place
    qg::pack24_tc_kernel<<<dim3((N + 255) / 256, K / 128), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        vals, K, N, vals_tc);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_gemm_w4a16_24_tc(const void* X, qg_dtype xdt, int M, int K, int N, const uint32_t* vals_tc,
                              const uint32_t* meta, const uint16_t* scales, const uint8_t* zeros, int group, void* Y,
                              void* workspace, size_t ws_bytes, qg_stream_t stream)
{
    if (xdt != QG_F16 && xdt != QG_BF16) return QG_ERR_DTYPE;
    if (M < 0 || K < 128 || K % 128 || N < 32 || N % 32 || group != 128) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!X || !vals_tc || !meta || !scales || !zeros || !Y || !workspace) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(vals_tc) || misaligned(meta) || misaligned(scales) || misaligned(zeros) ||
        misaligned(Y) || misaligned(workspace))
        return QG_ERR_ALIGN;
    if (ws_bytes < qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N)) return QG_ERR_WORKSPACE;
    const uint16_t* x = static_cast<const uint16_t*>(X);
    uint16_t* y = static_cast<uint16_t*>(Y);
    for (int m0 = 0; m0 < M; m0 += 32) {
        qg::SkinnyParams q{x + (int64_t)m0 * K, vals_tc, scales, zeros, y + (int64_t)m0 * N, std::min(32, M - m0), K, N};
        qg_status st;
        if (xdt == QG_BF16) {
            if (q.M <= 8) st = launch_w4a16_decode<1, true, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
            else if (q.M <= 16) st = launch_w4a16_decode<2, true, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
            else st = launch_w4a16_decode<4, true, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
        } else {
            if (q.M <= 8) st = launch_w4a16_decode<1, false, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
            else if (q.M <= 16) st = launch_w4a16_decode<2, false, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
            else st = launch_w4a16_decode<4, false, true>(q, vals_tc, scales, zeros, workspace, stream, meta);
        }
        if (st != QG_OK) return st;
    }
    return QG_OK;
}

qg_status qg_gptq(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group, double damp,
                  uint8_t* codes, uint16_t* scales, uint8_t* zeros, void* workspace, size_t ws_bytes,
                  qg_stream_t stream)
{
    if (!Xcal || !W || !codes || !scales || !zeros || !workspace) return QG_ERR_NULL;
    if (Mc < 1 || K < 8 || K > 16384 || N < 1 || group < 8 || group > 1024 || group % 8 || K % group ||
        !(damp > 0.0 && damp < 1e30))
        return QG_ERR_SHAPE;
    if (misaligned(Xcal) || misaligned(W) || misaligned(codes) || misaligned(scales) || misaligned(zeros) ||
        misaligned(workspace))
        return QG_ERR_ALIGN;
    if (ws_bytes < gptq_carve(nullptr, K, N).bytes) return QG_ERR_WORKSPACE;
    const GptqWs w = gptq_carve(workspace, K, N);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int kb = (K + 255) / 256, nb = (N + 255) / 256;
    // H, then its inverse by Gauss-Jordan (w.a is destroyed, w.inv receives H^-1)
    qg::gptq_hessian_kernel<<<dim3(kb, K), 256, 0, st>>>(Xcal, Mc, K, w.a);
    QG_CUDA(cudaGetLastError());
    qg::gptq_ridge_kernel<<<1, 32, 0, st>>>(w.a, K, damp);
    QG_CUDA(cudaGetLastError());
    qg::gptq_identity_kernel<<<dim3(kb, K), 256, 0, st>>>(w.inv, K);
    QG_CUDA(cudaGetLastError());
    for (int c = 0; c < K; ++c) {
        qg::gj_column_kernel<<<kb, 256, 0, st>>>(w.a, K, c, w.f);
        qg::gj_scale_kernel<<<kb, 256, 0, st>>>(w.a, w.inv, K, c, w.f);
        qg::gj_eliminate_kernel<<<dim3(kb, K), 256, 0, st>>>(w.a, w.inv, K, c, w.f);
    }
    QG_CUDA(cudaGetLastError());
    // the rows, in order
    const int64_t total = (int64_t)K * N;
    qg::gptq_load_kernel<<<(int)std::min<int64_t>((total + 255) / 256, 8 * num_sms()), 256, 0, st>>>(W, total, w.wc);
    QG_CUDA(cudaGetLastError());
    for (int k = 0; k < K; ++k) {
        if (k % group == 0)
            qg::gptq_group_kernel<<<nb, 256, 0, st>>>(w.wc, N, k, group, scales, zeros, w.s_col, w.z_col);
        qg::gptq_row_kernel<<<nb, 256, 0, st>>>(w.wc, K, N, k, w.inv, w.s_col, w.z_col, codes, w.e);
        const int rest = K - k - 1;
        if (rest > 0) {
            qg::gptq_update_kernel<<<dim3(nb, rest), 256, 0, st>>>(w.wc, K, N, k, w.inv, w.e);
            qg::gptq_eliminate_kernel<<<dim3((rest + 255) / 256, rest), 256, 0, st>>>(w.inv, K, k);
        }
    }
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_gptq_blocked(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group, double damp,
                          uint8_t* codes, uint16_t* scales, uint8_t* zeros, void* workspace, size_t ws_bytes,
                          qg_stream_t stream)
{
    if (!Xcal || !W || !codes || !scales || !zeros || !workspace) return QG_ERR_NULL;
    if (Mc < 1 || K < 8 || K > 16384 || N < 1 || group < 8 || group > 1024 || group % 8 || K % group ||
        !(damp > 0.0 && damp < 1e30))
        return QG_ERR_SHAPE;
    if (misaligned(Xcal) || misaligned(W) || misaligned(codes) || misaligned(scales) || misaligned(zeros) ||
        misaligned(workspace))
        return QG_ERR_ALIGN;
    if (ws_bytes < gptq_blocked_carve(nullptr, Mc, K, N).bytes) return QG_ERR_WORKSPACE;
    const GptqBlockedWs w = gptq_blocked_carve(workspace, Mc, K, N);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    constexpr int NB = qg::kCholNb;
    const int grid_ew = std::max(1, 8 * num_sms());
    // Hr = (2/Mc) Xr^T Xr (lower triangle), then the ridge on its diagonal
    const int64_t xt = (int64_t)Mc * K;
    qg::gptq_xrev_kernel<<<(int)std::min<int64_t>((xt + 255) / 256, grid_ew), 256, 0, st>>>(Xcal, Mc, K, w.xr);
    QG_CUDA(cudaGetLastError());
    qg_status r = dgemm<64, 64>({K, K, Mc, 2.0 / Mc, 0.0, w.xr, 1, K, w.xr, K, 1, w.a, K, 1, 0}, st);
    if (r != QG_OK) return r;
    qg::gptq_ridge_kernel<<<1, 32, 0, st>>>(w.a, K, damp);
    QG_CUDA(cudaGetLastError());
    // Lr: right-looking blocked Cholesky, 64-wide panels
    for (int p = 0; p < K; p += NB) {
        const int nb = std::min(NB, K - p), rows = K - p - nb;
        qg::chol_diag_kernel<<<1, 256, 0, st>>>(w.a, K, p, nb, w.dinv);
        QG_CUDA(cudaGetLastError());
        if (rows > 0) {
            qg::chol_panel_kernel<<<(rows + 127) / 128, 128, 0, st>>>(w.a, K, p, nb, w.dinv);
            QG_CUDA(cudaGetLastError());
            double* pan = w.a + (int64_t)(p + nb) * K + p;
            r = dgemm<64, 64>({rows, rows, nb, -1.0, 1.0, pan, K, 1, pan, 1, K, pan + nb, K, 1, 0}, st);
            if (r != QG_OK) return r;
        }
    }
    // Lr^-1 by block rows (its upper triangle stays zero)
    QG_CUDA(cudaMemsetAsync(w.inv, 0, 8 * (size_t)K * K, st));
    for (int r0 = 0; r0 < K; r0 += NB) {
        const int nb = std::min(NB, K - r0);
        if (r0 > 0) {
            r = dgemm<32, 32>({nb, r0, r0, 1.0, 0.0, w.a + (int64_t)r0 * K, K, 1, w.inv, K, 1, w.inv + (int64_t)r0 * K, K,
                               0, 1},
                              st);
            if (r != QG_OK) return r;
        }
        qg::trinv_rows_kernel<<<(r0 + nb + 127) / 128, 128, 0, st>>>(w.inv, K, r0, nb, w.dinv);
        QG_CUDA(cudaGetLastError());
    }
    // the rows, one group-sized block at a time; U[i][j] = Lr^-1[K-1-i][K-1-j]
    const int64_t total = (int64_t)K * N;
    qg::gptq_load_kernel<<<(int)std::min<int64_t>((total + 255) / 256, grid_ew), 256, 0, st>>>(W, total, w.wc);
    QG_CUDA(cudaGetLastError());
    const int NC = group <= 256 ? 32 : 8;
    const size_t smem = (size_t)group * NC * 8;
    static KernelInfo block_info;
    int occ = 0;
    r = prepare_kernel(block_info, qg::gptq_block_kernel, NC * 8, 64 * 1024, &occ);
    if (r != QG_OK) return r;
    for (int b = 0; b < K; b += group) {
        qg::gptq_block_kernel<<<(N + NC - 1) / NC, NC * 8, smem, st>>>(w.wc, K, N, b, group, w.inv, codes, scales,
                                                                        zeros, w.err, NC);
        QG_CUDA(cudaGetLastError());
        const int rest = K - b - group;
        if (rest > 0) {
            const double* ub = w.inv + (int64_t)(K - 1 - b) * K + (K - 1 - b - group);
            r = dgemm<64, 64>({rest, N, group, -1.0, 1.0, ub, -1, -(int64_t)K, w.err, N, 1,
                               w.wc + (int64_t)(b + group) * N, N, 0, 0},
                              st);
            if (r != QG_OK) return r;
        }
    }
    return QG_OK;
}

qg_status qg_awq_act_mean(const uint16_t* Xcal, int Mc, int K, float* xm, qg_stream_t stream)
{
    if (!Xcal || !xm) return QG_ERR_NULL;
    if (Mc < 1 || K < 1) return QG_ERR_SHAPE;
    if (misaligned(Xcal) || misaligned(xm)) return QG_ERR_ALIGN;
    qg::awq_act_mean_kernel<<<(K + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(Xcal, Mc, K, xm);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_awq_scales(const float* xm, int K, double alpha, float* s, float* inv_s, qg_stream_t stream)
{
    if (!xm || !s || !inv_s) return QG_ERR_NULL;
    if (K < 1 || !(alpha >= 0.0 && alpha <= 1.0)) return QG_ERR_SHAPE;
    if (misaligned(xm) || misaligned(s) || misaligned(inv_s)) return QG_ERR_ALIGN;
    qg::awq_scales_kernel<<<(K + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(xm, K, alpha, nullptr,
                                                                                                  0, s, inv_s);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_awq_scale_act(const uint16_t* X, int M, int K, const float* inv_s, uint16_t* Xs, qg_stream_t stream)
{
    if (M < 0 || K < 8 || K % 8) return QG_ERR_SHAPE;
    if (M == 0) return QG_OK;
    if (!X || !inv_s || !Xs) return QG_ERR_NULL;
    if (misaligned(X) || misaligned(inv_s) || misaligned(Xs)) return QG_ERR_ALIGN;
    const int64_t total8 = (int64_t)M * K / 8;
    const int grid = (int)std::min<int64_t>((total8 + 255) / 256, 8 * num_sms());
    qg::awq_scale_act_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(X, total8, K, inv_s, Xs);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_awq_search(const uint16_t* Xcal, int Mc, int K, const float* W, int N, int group, int n_grid,
                        double* mse, int32_t* best, float* s, float* inv_s, void* workspace, size_t ws_bytes,
                        qg_stream_t stream)
{
    if (!Xcal || !W || !mse || !best || !s || !inv_s || !workspace) return QG_ERR_NULL;
    if (Mc < 1 || K < 128 || K % 128 || N < 8 || N % 8 || group != 128 || n_grid < 1 || n_grid > 1024)
        return QG_ERR_SHAPE;
    if (misaligned(Xcal) || misaligned(W) || misaligned(mse) || misaligned(best) || misaligned(s) ||
        misaligned(inv_s) || misaligned(workspace))
        return QG_ERR_ALIGN;
    if (ws_bytes < awq_carve(nullptr, Mc, K, N).bytes) return QG_ERR_WORKSPACE;
    const AwqWs w = awq_carve(workspace, Mc, K, N);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int kgrid = (K + 255) / 256;
    const int64_t outs = (int64_t)Mc * N;
    qg_status r;
    // statistic and reference output, once
    qg::awq_act_mean_kernel<<<kgrid, 256, 0, st>>>(Xcal, Mc, K, w.xm);
    QG_CUDA(cudaGetLastError());
    qg::awq_ref_gemm_kernel<<<dim3((N + qg::kAwqRefBN - 1) / qg::kAwqRefBN, (Mc + qg::kAwqRefBM - 1) / qg::kAwqRefBM),
                              256, 0, st>>>(Xcal, W, Mc, K, N, w.yref);
    QG_CUDA(cudaGetLastError());
    // one candidate per grid point: scales -> Q(diag(s) W) -> packed -> X / s -> W4A16 GEMM -> error
    for (int i = 0; i < n_grid; ++i) {
        const double alpha = n_grid > 1 ? (double)i / (double)(n_grid - 1) : 0.0;
        qg::awq_scales_kernel<<<kgrid, 256, 0, st>>>(w.xm, K, alpha, nullptr, 0, w.sc, w.inv);
        QG_CUDA(cudaGetLastError());
        if ((r = qg_quantize_w4_group(W, w.sc, K, N, 128, 0, w.codes, w.scales, w.zeros, stream)) != QG_OK) return r;
        if ((r = qg_pack_nibbles(w.codes, K, N, w.packed, stream)) != QG_OK) return r;
        if ((r = qg_awq_scale_act(Xcal, Mc, K, w.inv, w.xs, stream)) != QG_OK) return r;
        if ((r = qg_gemm_w4a16(w.xs, QG_BF16, Mc, K, N, w.packed, w.scales, w.zeros, 128, w.yq, nullptr, 0, stream)) !=
            QG_OK)
            return r;
        qg::awq_sqerr_kernel<<<qg::kAwqErrBlocks, 256, 0, st>>>(w.yref, w.yq, outs, w.partials);
        QG_CUDA(cudaGetLastError());
        qg::awq_mse_finish_kernel<<<1, 32, 0, st>>>(w.partials, outs, mse + i);
        QG_CUDA(cudaGetLastError());
    }
    // the winner and its scales
    qg::awq_argmin_kernel<<<1, 32, 0, st>>>(mse, n_grid, best);
    QG_CUDA(cudaGetLastError());
    qg::awq_scales_kernel<<<kgrid, 256, 0, st>>>(w.xm, K, 0.0, best, n_grid, s, inv_s);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_quantize_w8_channel(const float* W, const float* s, int K, int N, int8_t* Wq, float* sw,
                                 qg_stream_t stream)
{
    if (!W || !Wq || !sw) return QG_ERR_NULL;
    if (K < 1 || N < 1) return QG_ERR_SHAPE;
    if (misaligned(W) || misaligned(s) || misaligned(Wq) || misaligned(sw)) return QG_ERR_ALIGN;
    if (N % 4 == 0) {
        // two streaming passes (absmax through sw as integer bits, then quantize), then
        // sw = absmax / 127 in place
        cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
        QG_CUDA(cudaMemsetAsync(sw, 0, sizeof(float) * (size_t)N, st));
        const dim3 grid((N + 127) / 128, (K + 255) / 256);
        unsigned int* amax = reinterpret_cast<unsigned int*>(sw);
        qg::w8_absmax_kernel<<<grid, 256, 0, st>>>(W, s, K, N, amax);
        QG_CUDA(cudaGetLastError());
        qg::w8_quant_kernel<<<grid, 256, 0, st>>>(W, s, K, N, amax, Wq);
        QG_CUDA(cudaGetLastError());
        qg::w8_scale_kernel<<<(N + 255) / 256, 256, 0, st>>>(sw, N);
        QG_CUDA(cudaGetLastError());
        return QG_OK;
    }
    qg::quantize_w8_channel_kernel<<<(N + 127) / 128, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, s, K, N,
                                                                                                          Wq, sw);
    QG_CUDA(cudaGetLastError());
    return QG_OK;
}

qg_status qg_selftest_bounded_wait(uint64_t limit_ns, qg_stream_t stream)
{
    unsigned long long lim = limit_ns ? (unsigned long long)limit_ns : 2000000000ull;
    unsigned long long saved = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    QG_CUDA(cudaMemcpyFromSymbol(&saved, qg::g_wait_limit_ns, sizeof(saved)));
    QG_CUDA(cudaMemcpyToSymbolAsync(qg::g_wait_limit_ns, &lim, sizeof(lim), 0, cudaMemcpyHostToDevice, st));
    qg::selftest_wait_kernel<<<1, 32, 0, st>>>();
    QG_CUDA(cudaGetLastError());
    QG_CUDA(cudaMemcpyToSymbolAsync(qg::g_wait_limit_ns, &saved, sizeof(saved), 0, cudaMemcpyHostToDevice, st));
    QG_CUDA(cudaStreamSynchronize(st));
    return QG_OK;
}

}  // extern "C"

// ===========================================================================
// Allocation-free W4A16 entry point
//
// Some callers cannot call cudaMalloc (or torch's allocator) at the point where they
// run a GEMM: code being captured into a CUDA graph (allocation is not allowed
// inside a capture), plugins and custom operators inside a host framework that owns
// every device allocation and gives the operator no allocator, and latency-bound
// paths where an allocation's implicit device synchronisation is unacceptable.
// For them the decode kernel's scratch (the partial tiles of split column slabs) lives
// in one statically sized device array instead of a caller workspace.
// ===========================================================================
namespace {

// 6 MiB per GPU that loads this library, held until the process exits.  A decode
// launch of 32 tokens needs, per CTA (at most one per SM), an 8-byte token and one
// partial tile of 128 x 32 fp32 (16 KiB): 2.4 MiB on a 148-SM B200, and the array
// covers GPUs of up to 380 SMs.
constexpr size_t kNoAllocScratchBytes = size_t(6) << 20;
static __device__ __align__(256) unsigned char qg_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array, per device.  In host code the array's name is only a
// host-side stand-in, so the address must come from cudaGetSymbolAddress, called
// with the device current.  Cached per device slot (atomic: first calls from several
// host threads store the same address); a device beyond the slots queries each time.
std::atomic<void*> g_noalloc_addr[kMaxDevices];

qg_status noalloc_scratch(void** out)
{
    int dev = 0;
    qg_status st = current_device(&dev);
    if (st != QG_OK) return st;
    if (cached_slot(dev)) {
        void* p = g_noalloc_addr[dev].load(std::memory_order_acquire);
        if (p) {
            *out = p;
            return QG_OK;
        }
    }
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, qg_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(qg_noalloc_scratch)");
    if (cached_slot(dev)) g_noalloc_addr[dev].store(ptr, std::memory_order_release);
    *out = ptr;
    return QG_OK;
}

}  // namespace

extern "C" qg_status qg_gemm_w4a16_noalloc(const void* X, qg_dtype xdt, int M, int K, int N,
                                           const uint32_t* packed, const uint16_t* scales, const uint8_t* zeros,
                                           int group, void* Y, qg_stream_t stream)
{
    const size_t need = qg_workspace_size(QG_OP_GEMM_W4A16, M, K, N);
    if (need == 0)  // no scratch used for this shape (or invalid arguments): plain call
        return qg_gemm_w4a16(X, xdt, M, K, N, packed, scales, zeros, group, Y, nullptr, 0, stream);
    if (need > kNoAllocScratchBytes) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "qg_gemm_w4a16_noalloc: this shape needs %zu bytes of scratch, the static buffer holds %zu", need,
                 kNoAllocScratchBytes);
        return QG_ERR_WORKSPACE;
    }
    if (xdt != QG_F16 && xdt != QG_BF16) return QG_ERR_DTYPE;
    if (!X || !packed || !scales || !zeros || !Y) return QG_ERR_NULL;
    if (group != 128) return QG_ERR_SHAPE;
    if (misaligned(X) || misaligned(packed) || misaligned(scales) || misaligned(zeros) || misaligned(Y))
        return QG_ERR_ALIGN;
    void* ws = nullptr;
    qg_status st = noalloc_scratch(&ws);
    if (st != QG_OK) return st;
    // A partial tile is read only after its token (unique to the launch) is seen, and
    // every launch clears the tokens it consumed, so nothing in the array has to start
    // at zero; it keeps the last call's contents.
    return qg_gemm_w4a16(X, xdt, M, K, N, packed, scales, zeros, group, Y, ws, kNoAllocScratchBytes, stream);
}
