// Host-side launch helpers.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace la {

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute is per device context). Safe to call on every launch. The
// kernel is a template argument so that each kernel keeps its own flag.
template <auto kernel>
cudaError_t ensure_smem(size_t bytes) {
    static std::atomic<uint64_t> done{0};
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

}  // namespace la
