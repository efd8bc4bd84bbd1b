// Test probe for the library's bounded waits (csrc/tc_common.cuh): one CTA,
// two warps, each waiting on an mbarrier that nothing ever arrives at.
// Warp 0's wait must expire (timeout bit in *err, abort flag set); warp 1's
// wait must then return early because of the CTA abort flag. Each warp's
// lane 0 records its result and how long it waited.
#include "tc_common.cuh"

using namespace la::tc;

__global__ void wait_timeout_kernel(uint32_t* err, unsigned long long* result) {
    __shared__ uint64_t bars[2];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        cta_abort_reset();
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (lane == 0) {
        const unsigned long long t0 = globaltimer();
        // warp 1 starts a little later, so that warp 0's wait expires first
        if (warp == 1) {
            while (globaltimer() - t0 < 500000000ull) {
            }
        }
        const unsigned long long t1 = globaltimer();
        const bool ok = mbar_wait(&bars[warp], 0, err);
        result[2 * warp] = ok ? 1ull : 0ull;
        result[2 * warp + 1] = globaltimer() - t1;
    }
    __syncthreads();
}

extern "C" int wait_timeout_probe(uint32_t* err, unsigned long long* result) {
    wait_timeout_kernel<<<1, 64>>>(err, result);
    return (int)cudaGetLastError();
}
