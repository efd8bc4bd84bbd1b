// la_kv_summary_static: the KV summary with its scratch in a fixed device
// array owned by the library, for callers that cannot allocate device memory
// (see include/la.h).

#include <cudaTypedefs.h>
#include <la.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "tc_common.cuh"

namespace la {
namespace {

// Largest workspace la_kv_summary_static serves (partial state records plus
// the error word). Every GPU that loads the library holds this array until
// the process exits.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch in each CUDA context, looked up once per
// context with it current. The host-side symbol is only a handle: it must
// never be passed to a kernel. Keyed by the context's unique id rather than
// the device ordinal: a device reset (or a context the caller created with
// the driver API) loads the module again, and the array can move.
std::mutex g_mutex;
struct CtxAddr {
    unsigned long long ctx;
    void* addr;
};
CtxAddr g_addr[64];  // the most recent contexts first seen, oldest replaced first
int g_naddr = 0;

struct CtxApi {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxApi& ctx_api() {
    static CtxApi api;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    return api;
}

// Id of the current context, 0 if there is none yet.
unsigned long long current_ctx_id() {
    const CtxApi& api = ctx_api();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (api.get_current == nullptr || api.get_id == nullptr) return 0;
    if (api.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (api.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

la_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    unsigned long long id = current_ctx_id();
    if (id != 0) {
        for (int i = 0; i < std::min(g_naddr, 64); ++i)
            if (g_addr[i].ctx == id) {
                *out = g_addr[i].addr;
                return LA_OK;
            }
    }
    // first call in this context (the lookup also makes the runtime's
    // context current when none was yet)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (id == 0) id = current_ctx_id();
    if (id != 0) g_addr[g_naddr++ % 64] = CtxAddr{id, p};
    *out = p;
    return LA_OK;
}

// After the KV summary: if one of its bounded waits expired (the error word
// at the start of the array has FLAG_TIMEOUT set), fill S and z with NaN, so
// that the failure shows in the caller's outputs (this entry point has no
// workspace the caller could pass to la_last_error).
__global__ void nan_on_timeout_kernel(const uint32_t* __restrict__ err, float* __restrict__ S, long long nS,
                                      float* __restrict__ z, long long nz) {
    if ((*reinterpret_cast<const volatile uint32_t*>(err) & tc::FLAG_TIMEOUT) == 0) return;
    const float nan = __int_as_float(0x7fc00000);
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nS; i += stride) S[i] = nan;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nz; i += stride) z[i] = nan;
}

}  // namespace
}  // namespace la

extern "C" la_status la_kv_summary_static(const la_desc* desc, const void* k, const void* v,
                                          float* S_out, float* z_out, void* stream) {
    // the descriptor and pointers first, as la_kv_summary checks them, before any CUDA call
    const la_status arg = la::kv_summary_args(desc, k, v, S_out, z_out);
    if (arg != LA_OK) return arg;
    const size_t need = la_workspace_size(desc, LA_OP_KV_SUMMARY, 0);
    if (need == 0 || need > la::kStaticScratchBytes) return LA_ERR_WORKSPACE;
    void* ws = nullptr;
    const la_status st = la::scratch_address(&ws);
    if (st != LA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the error word must start at zero; the rest of the scratch needs no clearing
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    const la_status r = la::kv_summary_checked(desc, k, v, S_out, z_out, ws, la::kStaticScratchBytes, s);
    if (r != LA_OK) return r;
    const long long bh = (long long)desc->B * desc->H;
    la::nan_on_timeout_kernel<<<32, 256, 0, s>>>(static_cast<const uint32_t*>(ws), S_out,
                                                  bh * desc->d * desc->d, z_out, bh * desc->d);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    return LA_OK;
}
