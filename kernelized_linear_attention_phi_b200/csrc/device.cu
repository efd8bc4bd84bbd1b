// Device queries behind the work plans (device.h).

#include <cuda_runtime.h>

#include <mutex>

#include "device.h"

namespace la {
namespace {

constexpr int kDefaultSms = 148;  // a full B200, for sizing without a device

std::mutex g_mutex;
int g_sms[64] = {};
// answers of max_active_clusters (a handful of launch shapes per device)
struct ClusterAnswer {
    int dev, cluster, threads;
    size_t smem;
    int n;
};
ClusterAnswer g_clusters[64];
int g_nclusters = 0;

// A kernel with no registers or shared memory of its own to speak of: its
// occupancy is bound only by the launch shape the query gives it.
__global__ void occupancy_shape_kernel() {}

}  // namespace

int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return kDefaultSms;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            return kDefaultSms;
        }
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

int max_active_clusters(int cluster, int threads, size_t smem) {
    int dev = 0;
    if (cluster <= 0 || threads <= 0 || cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    for (int i = 0; i < g_nclusters; ++i) {
        const ClusterAnswer& a = g_clusters[i];
        if (a.dev == dev && a.cluster == cluster && a.threads == threads && a.smem == smem) return a.n;
    }
    int n = 0;
    cudaError_t e = cudaFuncSetAttribute(occupancy_shape_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e == cudaSuccess && cluster > 8)
        e = cudaFuncSetAttribute(occupancy_shape_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)cluster);
        cfg.blockDim = dim3((unsigned)threads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&n, occupancy_shape_kernel, &cfg);
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return 0;  // not cached: a later call may succeed
    }
    if (g_nclusters < 64) g_clusters[g_nclusters++] = ClusterAnswer{dev, cluster, threads, smem, n};
    return n;
}

}  // namespace la
