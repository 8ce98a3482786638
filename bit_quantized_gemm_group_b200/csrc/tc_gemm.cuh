// tc_gemm.cuh -- tcgen05 (TMEM accumulator, TMA-fed) tile kernels for prefill shapes.
#pragma once
#include <climits>

#include "../../include/qgemm.h"
#include "common.cuh"

namespace qg {

// Smallest M routed to the tensor-memory tile kernels (smaller M uses the skinny paths).
constexpr int kTcMinM = INT_MAX;

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

inline qg_status tc_w4a16_launch(const TcW4A16Args&, qg_stream_t) { return QG_ERR_UNSUPPORTED; }
inline qg_status tc_w8a8_launch(const TcInt8Args&, qg_stream_t) { return QG_ERR_UNSUPPORTED; }
inline qg_status tc_w4a8_launch(const TcInt8Args&, qg_stream_t) { return QG_ERR_UNSUPPORTED; }

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
