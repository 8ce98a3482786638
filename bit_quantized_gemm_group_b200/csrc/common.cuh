// common.cuh -- device helpers shared by the kernels of libqgemm.so (sm_100a only).
//
// Sticky status word, bf16/fp16 bit helpers, and thin inline-PTX wrappers for the
// Blackwell machinery the tile kernels use: mbarriers with bounded waits, TMA tiled
// loads, tcgen05 (TMEM alloc / MMA / commit / load) and cluster DSMEM access.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define QG_DEV_INLINE __device__ __forceinline__

namespace qg {

// ---------------------------------------------------------------------------
// Device status word (per device, sticky until qg_device_status() reads it).
// Values are qg_status codes; the first error recorded wins.
// ---------------------------------------------------------------------------
__device__ unsigned int g_status;
// Bounded waits give up after this many nanoseconds (set by the host).
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

QG_DEV_INLINE void set_status(unsigned int code) { atomicCAS(&g_status, 0u, code); }

QG_DEV_INLINE unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// 16-bit float bit helpers
// ---------------------------------------------------------------------------
// Exact int32 -> fp32 for |v| < 2^22 on the full-rate pipes (integer add, fp32 add):
// add into the mantissa of 1.5 * 2^23, subtract it back.  (The conversion instruction
// itself issues at a fraction of the fp32 rate.)
QG_DEV_INLINE float i2f_small(uint32_t v) { return __uint_as_float(v + 0x4B400000u) - 12582912.0f; }

QG_DEV_INLINE float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

QG_DEV_INLINE uint32_t pack_bf16x2_rn(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

QG_DEV_INLINE uint32_t pack_f16x2_rn(float lo, float hi)
{
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

QG_DEV_INLINE uint16_t f32_to_bf16_bits(float x)
{
    __nv_bfloat16 v = __float2bfloat16_rn(x);
    return *reinterpret_cast<uint16_t*>(&v);
}

QG_DEV_INLINE uint16_t f32_to_f16_bits(float x)
{
    __half v = __float2half_rn(x);
    return *reinterpret_cast<uint16_t*>(&v);
}

QG_DEV_INLINE uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv)
{
    // (a & mask) | orv in one LOP3
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
    return r;
}

QG_DEV_INLINE uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// ---------------------------------------------------------------------------
// Global loads
// ---------------------------------------------------------------------------
QG_DEV_INLINE uint4 ldg_stream_v4(const void* p)
{
    // read-once data: do not keep it in L1
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

QG_DEV_INLINE uint4 ldg_v4(const void* p)
{
    uint4 v;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers (bounded waits), fences
// ---------------------------------------------------------------------------
QG_DEV_INLINE uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

QG_DEV_INLINE void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

QG_DEV_INLINE void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

QG_DEV_INLINE void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

QG_DEV_INLINE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

QG_DEV_INLINE bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the barrier's phase with the given parity has completed.  Gives up
// after g_wait_limit_ns: records QG_ERR_TIMEOUT (7) and returns false; the caller
// then winds down without touching the pipeline again.
QG_DEV_INLINE bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    const unsigned long long lim = g_wait_limit_ns;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u && globaltimer_ns() - t0 > lim) {
            set_status(7u);
            return false;
        }
    }
}

// Same bounded wait, but backing off with nanosleep between polls (32 ns doubling to
// 256 ns).  For roles with many warps waiting at once (epilogue, dequant, consumers):
// their polling then leaves the issue slots to the warps doing the work.
QG_DEV_INLINE bool mbar_wait_backoff(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    const unsigned long long lim = g_wait_limit_ns;
    uint32_t ns = 32;
    for (uint32_t it = 1;; ++it) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (ns < 256) ns <<= 1;
        if ((it & 15u) == 0u && globaltimer_ns() - t0 > lim) {
            set_status(7u);
            return false;
        }
    }
}

QG_DEV_INLINE unsigned long long ld_acquire_u64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

QG_DEV_INLINE void st_release_u64(unsigned long long* p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Split-slab pieces between the CTAs of one decode launch: a CTA publishes its piece's
// partial tile under the launch's 64-bit token (never 0); the CTA that finishes the slab
// watches the tokens of CTAs c_first .. c_last with the lanes of one warp (all polls in
// flight at once), bounded: false (and QG_ERR_TIMEOUT recorded) if one never appears.
QG_DEV_INLINE bool watch_tokens(const unsigned long long* flags, int c_first, int c_last, unsigned long long token,
                                int lane)
{
    const unsigned long long t0 = globaltimer_ns();
    const unsigned long long lim = g_wait_limit_ns;
    for (int i0 = c_first; i0 <= c_last; i0 += 32) {
        const int c = i0 + lane;
        bool seen = c > c_last;  // lanes past the last piece have nothing to watch
        for (uint32_t it = 0;; ++it) {
            if (!seen) seen = ld_acquire_u64(flags + c) == token;
            if (__all_sync(0xffffffffu, seen)) break;
            __nanosleep(32);
            if ((it & 15u) == 15u && globaltimer_ns() - t0 > lim) {
                if (lane == 0) set_status(7u);
                return false;
            }
        }
    }
    return true;
}

// Named barrier `id` over `count` threads that also ANDs a predicate across them.
QG_DEV_INLINE int named_bar_and(uint32_t id, uint32_t count, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(count)
        : "memory");
    return (int)r;
}

QG_DEV_INLINE void named_bar_sync(uint32_t id, uint32_t count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Arrive on named barrier `id` without waiting (the threads that bar.sync on it wait for
// `count` arrivals in all); the caller's earlier shared-memory writes are visible to them.
QG_DEV_INLINE void named_bar_arrive(uint32_t id, uint32_t count)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

QG_DEV_INLINE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------
// TMA (tiled tensor loads into shared memory, completion on an mbarrier)
// ---------------------------------------------------------------------------
QG_DEV_INLINE void tma_prefetch_desc(const CUtensorMap* m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

QG_DEV_INLINE void tma_load_2d(const CUtensorMap* m, uint64_t* bar, void* smem_dst, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

QG_DEV_INLINE void tma_load_3d(const CUtensorMap* m, uint64_t* bar, void* smem_dst, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, loads
// ---------------------------------------------------------------------------
QG_DEV_INLINE void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

QG_DEV_INLINE void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;"); }

QG_DEV_INLINE void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

QG_DEV_INLINE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
QG_DEV_INLINE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem]^T for one instruction shape; kind::f16 (bf16/fp16 in,
// fp32 out).  Lane i of A holds row i, and each 32-bit column holds two consecutive k
// values (so one K = 16 step spans 8 columns).
QG_DEV_INLINE void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
        : "memory");
}

// kind::i8 (int8 in, int32 out)
QG_DEV_INLINE void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accum)
        : "memory");
}

// kind::i8 with A (M x K, int8) read from tensor memory: four consecutive k per 32-bit column
QG_DEV_INLINE void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
QG_DEV_INLINE void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread
QG_DEV_INLINE void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns -> 16 registers per thread
QG_DEV_INLINE void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// 4-byte global -> shared copy that bypasses registers (zero-filled when !valid)
QG_DEV_INLINE void cp_async_4(void* dst_smem, const void* src, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst_smem)), "l"(src),
                 "r"(valid ? 4 : 0)
                 : "memory");
}
QG_DEV_INLINE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
QG_DEV_INLINE void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// 32 lanes x 1 32-bit column -> 1 register per thread
QG_DEV_INLINE uint32_t tmem_ld_32x32b_x1(uint32_t taddr)
{
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return r;
}

QG_DEV_INLINE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 16 registers per thread -> 32 lanes x 16 consecutive 32-bit columns
QG_DEV_INLINE void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

QG_DEV_INLINE void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, swizzle mode in bits 61-63
// (0 none, 2 = 128-byte swizzle).
QG_DEV_INLINE uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t swizzle_mode)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(swizzle_mode & 7) << 61;
    return d;
}

// ---------------------------------------------------------------------------
// Clusters and distributed shared memory
// ---------------------------------------------------------------------------
QG_DEV_INLINE uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

QG_DEV_INLINE void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// address of the same shared variable in CTA `rank` of this cluster
QG_DEV_INLINE uint32_t dsmem_addr(uint32_t local_saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_saddr), "r"(rank));
    return r;
}

QG_DEV_INLINE float ld_dsmem_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

}  // namespace qg
