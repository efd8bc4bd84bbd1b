// Prefix-mask query binning ("trim-transformer 0.1.0", "Masking": query i
// sees keys 0..m_i). Query i is answered at chunk floor((m_i + 1) / chunk):
// the state of the keys before that chunk plus a partial chunk of
// (m_i + 1) mod chunk keys.

#include "common.cuh"
#include "internal.h"
#include "launch_util.h"

namespace la {
namespace {

constexpr int kBinThreads = 1024;

// One CTA per sequence: clamp, histogram, exclusive scan, scatter.
__global__ void __launch_bounds__(kBinThreads)
bin_kernel(const int32_t* __restrict__ m, int N, int chunk, int nbins, int32_t* __restrict__ perm,
           int32_t* __restrict__ bin_start, int32_t* __restrict__ msort, uint32_t* __restrict__ flags) {
    extern __shared__ int32_t cnt[];  // nbins + 1
    __shared__ int32_t warp_tot[kBinThreads / 32];
    // Reads only the caller's mask and writes tables that no kernel of the
    // call reads before the block-state scan, which waits for this kernel:
    // launched after the KV pass, it runs beside it and waits for it only at
    // its end (below).
    pdl_launch_dependents();
    const int b = blockIdx.x;
    const int32_t* mb = m + (size_t)b * N;
    for (int c = threadIdx.x; c <= nbins; c += kBinThreads) cnt[c] = 0;
    __syncthreads();
    bool bad = false;
    for (int i = threadIdx.x; i < N; i += kBinThreads) {
        int32_t mi = mb[i];
        if (mi < 0 || mi > N - 1) {
            bad = true;
            mi = mi < 0 ? 0 : N - 1;
        }
        atomicAdd(&cnt[(mi + 1) / chunk], 1);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(flags, FLAG_MASK_RANGE);
    // exclusive scan of cnt[0..nbins) into cnt (cnt[nbins] becomes the total):
    // each thread scans a contiguous run, then the run totals are scanned.
    const int per = (nbins + kBinThreads) / kBinThreads;
    const int lo = threadIdx.x * per;
    const int hi = min(nbins + 1, lo + per);
    int32_t run = 0;
    for (int c = lo; c < hi; ++c) run += (c < nbins) ? cnt[c] : 0;
    // block-wide exclusive scan of `run`
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int32_t base = (wid > 0 ? warp_tot[wid - 1] : 0) + incl - run;
    for (int c = lo; c < hi; ++c) {
        const int32_t v = (c < nbins) ? cnt[c] : 0;
        cnt[c] = base;
        bin_start[(size_t)b * (nbins + 1) + c] = base;
        base += v;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += kBinThreads) {
        const int32_t mi = min(max(mb[i], 0), N - 1);
        const int pos = atomicAdd(&cnt[(mi + 1) / chunk], 1);
        perm[(size_t)b * N + pos] = i;
        msort[(size_t)b * N + pos] = mi;
    }
    // This grid does not complete before the KV pass it runs beside: a
    // kernel that waits for this one then finds both complete.
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

cudaError_t bin_queries(const Problem& p, const int32_t* m, int chunk, int nbins, int32_t* perm,
                        int32_t* bin_start, int32_t* msort, uint32_t* flags, cudaStream_t st) {
    const size_t smem = sizeof(int32_t) * (size_t)(nbins + 1);
    cudaError_t e = ensure_smem<bin_kernel>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(bin_kernel, dim3(p.B), dim3(kBinThreads), smem, st, m, p.N, chunk, nbins, perm,
                      bin_start, msort, flags);
}

}  // namespace la
