// Per-launch timing of the library's calls (la_timing_enable / la_timing_read):
// a measurement aid for callers that want each kernel's share of a call, for
// example a benchmark that divides a kernel's algorithmic bytes by its own
// duration. While enabled, every entry point records one CUDA event on its
// stream before its first kernel and one after each kernel it launches; the
// events are the library's own (created by la_timing_enable on the current
// device). Under stream capture the records become event nodes of the graph
// and are taken again at every replay.

#include <atomic>
#include <mutex>

#include "internal.h"
#include "launch_util.h"

namespace la {
namespace {

constexpr int kMaxMarks = 16;  // kernels timed per call at most

std::mutex g_mu;
std::atomic<bool> g_on{false};
int g_dev = -1;
cudaEvent_t g_ev[kMaxMarks + 1] = {};
int g_next = 0;  // events recorded so far by the current call
int g_last = 0;  // events recorded by the last call

// Under stream capture a plain record only marks a dependency; the
// "external" flag makes it an event node of the graph.
cudaError_t record(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return cudaGetLastError();
    return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal)
                                                : cudaEventRecord(ev, st);
}

}  // namespace

void timing_begin(cudaStream_t st) {
    if (!g_on.load(std::memory_order_acquire)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    g_next = record(g_ev[0], st) == cudaSuccess ? 1 : 0;
    g_last = g_next;
}

void timing_mark(cudaStream_t st) {
    if (!g_on.load(std::memory_order_acquire)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_next < 1 || g_next > kMaxMarks) return;
    if (record(g_ev[g_next], st) == cudaSuccess) g_last = ++g_next;
}

}  // namespace la

using namespace la;

extern "C" {

la_status la_timing_enable(int32_t enable) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!enable) {
        g_on.store(false, std::memory_order_release);
        return LA_OK;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (g_dev != dev) {
        for (int i = 0; i <= kMaxMarks; ++i) {
            if (g_ev[i] != nullptr) cudaEventDestroy(g_ev[i]);
            g_ev[i] = nullptr;
        }
        g_dev = -1;
        for (int i = 0; i <= kMaxMarks; ++i) {
            if (cudaEventCreate(&g_ev[i]) != cudaSuccess) {
                cudaGetLastError();
                return LA_ERR_CUDA;
            }
        }
        g_dev = dev;
    }
    g_next = g_last = 0;
    g_on.store(true, std::memory_order_release);
    return LA_OK;
}

la_status la_timing_read(float* ms, int32_t capacity, int32_t* count) {
    if (count == nullptr || capacity < 0 || (capacity > 0 && ms == nullptr)) return LA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_mu);
    *count = 0;
    if (g_last < 2) return LA_OK;
    if (cudaEventSynchronize(g_ev[g_last - 1]) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    const int n = g_last - 1;
    for (int i = 0; i < n && i < capacity; ++i) {
        if (cudaEventElapsedTime(&ms[i], g_ev[i], g_ev[i + 1]) != cudaSuccess) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
    }
    *count = n;
    return LA_OK;
}

}  // extern "C"
