// la_kv_summary_static: the KV summary with its scratch in a fixed device
// array owned by the library, for callers that cannot allocate device memory
// (see include/la.h).

#include <la.h>

#include <mutex>

#include "internal.h"

namespace la {
namespace {

// Largest workspace la_kv_summary_static serves (partial state records plus
// the error word). Every GPU that loads the library holds this array until
// the process exits.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on each device, looked up once per
// device with that device current. The host-side symbol is only a handle:
// it must never be passed to a kernel.
std::mutex g_mutex;
void* g_addr[64] = {};

la_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return LA_OK;
}

}  // namespace
}  // namespace la

extern "C" la_status la_kv_summary_static(const la_desc* desc, const void* k, const void* v,
                                          float* S_out, float* z_out, void* stream) {
    const size_t need = la_workspace_size(desc, LA_OP_KV_SUMMARY, 0);
    if (need == 0) {
        // invalid or unsupported: report exactly what la_kv_summary would
        return la::kv_summary_checked(desc, k, v, S_out, z_out, nullptr, 0,
                                      static_cast<cudaStream_t>(stream));
    }
    if (need > la::kStaticScratchBytes) return LA_ERR_WORKSPACE;
    void* ws = nullptr;
    const la_status st = la::scratch_address(&ws);
    if (st != LA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the error word must start at zero; the rest of the scratch needs no clearing
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return la::kv_summary_checked(desc, k, v, S_out, z_out, ws, la::kStaticScratchBytes, s);
}
