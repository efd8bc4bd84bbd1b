// CUDA-core (SIMT) kernels: every form, both element types, d in {16,32,64,128}.
//
// These are the fp32 path (fp32 inputs keep fp32 products, which the 1e-4
// tolerance needs) and the general fallback shape set. The bf16 hot paths for
// d = 64 and 128 run on the tensor cores (tc_*.cu).
//
// Math ("nx_f32_linear_attention.nx source", header comment and loops):
//   S = sum_j phi(K_j) (x) V_j,  z = sum_j phi(K_j),
//   out_i = phi(Q_i) S / (phi(Q_i) . z).
// Chunked causal / prefix forms ("trim-transformer 0.1.0", "Masking"): the
// queries answered at chunk c see the state of all keys before the chunk plus
// the keys of chunk c up to their own limit (i for causal, m_i for a prefix
// mask).

#include "common.cuh"
#include "internal.h"
#include "launch_util.h"

namespace la {
namespace {

constexpr int kThreads = 256;
constexpr int kTT = 32;  // tokens per shared-memory tile in kv_partial
constexpr int kC = 64;   // chunk length of the SIMT chunked kernel

template <int R>
__device__ __forceinline__ void lds(const float* p, float* o) {
    if constexpr (R % 4 == 0) {
#pragma unroll
        for (int i = 0; i < R / 4; ++i) {
            const float4 v = reinterpret_cast<const float4*>(p)[i];
            o[4 * i] = v.x; o[4 * i + 1] = v.y; o[4 * i + 2] = v.z; o[4 * i + 3] = v.w;
        }
    } else if constexpr (R == 2) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        o[0] = v.x; o[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < R; ++i) o[i] = p[i];
    }
}

// ---------------------------------------------------------------------------
// Partial KV summary over a token range of one head.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
kv_partial_kernel(const T* __restrict__ K, const T* __restrict__ V, int N, int tps, int nsplit,
                  int phi, float* __restrict__ part) {
    constexpr int R = D / 16;
    __shared__ __align__(16) float sK[kTT * D];
    __shared__ __align__(16) float sV[kTT * D];
    const int s = blockIdx.x;
    const long long bh = blockIdx.y;
    const int t0 = s * tps;
    const int t1 = min(N, t0 + tps);
    pdl_wait();
    const T* Kh = K + bh * (long long)N * D;
    const T* Vh = V + bh * (long long)N * D;
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;

    float acc[R][R];
    float zacc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        zacc[r] = 0.f;
#pragma unroll
        for (int c = 0; c < R; ++c) acc[r][c] = 0.f;
    }
    for (int base = t0; base < t1; base += kTT) {
        const int valid = min(kTT, t1 - base);
        tile_to_smem<T, D, D>(sK, Kh + (long long)base * D, kTT, valid, true, phi);
        tile_to_smem<T, D, D>(sV, Vh + (long long)base * D, kTT, valid, false, phi);
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < kTT; ++t) {
            float a[R], b[R];
            lds<R>(sK + t * D + ta * R, a);
            lds<R>(sV + t * D + tb * R, b);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                zacc[r] += a[r];
#pragma unroll
                for (int c = 0; c < R; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
            }
        }
        __syncthreads();
    }
    float* o = part + ((size_t)bh * nsplit + s) * (size_t)(D * D + D);
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int c = 0; c < R; ++c) o[(ta * R + r) * D + tb * R + c] = acc[r][c];
        if (tb == 0) o[D * D + ta * R + r] = zacc[r];
    }
}

// ---------------------------------------------------------------------------
// Fixed-order reductions of state records.
// ---------------------------------------------------------------------------
__global__ void state_reduce_kernel(const float* __restrict__ part, int nsplit, int D,
                                    float* __restrict__ S, float* __restrict__ z) {
    const int rec = D * D + D;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const long long bh = blockIdx.y;
    pdl_wait();
    if (e < rec) {
        const float* p = part + (size_t)bh * nsplit * rec + e;
        float s = 0.f;
        for (int i = 0; i < nsplit; ++i) s += p[(size_t)i * rec];
        if (e < D * D) S[(size_t)bh * D * D + e] = s;
        else z[(size_t)bh * D + (e - D * D)] = s;
    }
}

// One thread per float4 of a record; loads are issued eight blocks at a time
// so that several are in flight, the running sum stays in registers.
// With `reverse` the blocks are taken last to first (suffix sums).
__global__ void state_scan_kernel(float* __restrict__ part, int nblk, int D,
                                  float* __restrict__ S_total, float* __restrict__ z_total, int reverse) {
    const int rec4 = (D * D + D) / 4;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const long long bh = blockIdx.y;
    pdl_wait();
    if (e >= rec4) {
        return;
    }
    float4* p = reinterpret_cast<float4*>(part + (size_t)bh * nblk * (rec4 * 4)) + e;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int b0 = 0; b0 < nblk; b0 += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (b0 + j < nblk) v[j] = p[(size_t)(reverse ? nblk - 1 - (b0 + j) : b0 + j) * rec4];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (b0 + j < nblk) {
                p[(size_t)(reverse ? nblk - 1 - (b0 + j) : b0 + j) * rec4] = run;
                run.x += v[j].x;
                run.y += v[j].y;
                run.z += v[j].z;
                run.w += v[j].w;
            }
        }
    }
    if (S_total != nullptr) {
        const float r[4] = {run.x, run.y, run.z, run.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int idx = 4 * e + q;
            if (idx < D * D) S_total[(size_t)bh * D * D + idx] = r[q];
            else z_total[(size_t)bh * D + (idx - D * D)] = r[q];
        }
    }
}

// ---------------------------------------------------------------------------
// Readout: out_i = phi(q_i) S / (phi(q_i).z).
// ---------------------------------------------------------------------------
template <int D>
constexpr size_t readout_smem() {
    return sizeof(float) * ((size_t)D * D + D + 64 * (D + 4) + 64);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
readout_kernel(const T* __restrict__ Q, const float* __restrict__ S, const float* __restrict__ z,
               T* __restrict__ out, int N, int phi, int normalize) {
    constexpr int TQ = 64, LDQ = D + 4, RC = D / 16, RT = TQ / 16;
    extern __shared__ __align__(16) float sm[];
    float* sS = sm;
    float* sz = sS + D * D;
    float* sQ = sz + D;
    float* sDen = sQ + TQ * LDQ;
    const int tile = blockIdx.x;
    const long long bh = blockIdx.y;
    pdl_wait();
    const float4* S4 = reinterpret_cast<const float4*>(S + (size_t)bh * D * D);
    for (int e = threadIdx.x; e < D * D / 4; e += kThreads) reinterpret_cast<float4*>(sS)[e] = S4[e];
    for (int e = threadIdx.x; e < D; e += kThreads) sz[e] = z[(size_t)bh * D + e];
    const int row0 = tile * TQ;
    const T* Qh = Q + bh * (long long)N * D;
    tile_to_smem<T, D, LDQ>(sQ, Qh + (long long)row0 * D, TQ, min(TQ, N - row0), true, phi);
    __syncthreads();
    if (normalize && threadIdx.x < TQ) {
        float den = 0.f;
        for (int a = 0; a < D; ++a) den = fmaf(sQ[threadIdx.x * LDQ + a], sz[a], den);
        sDen[threadIdx.x] = den;
    }
    const int tc = threadIdx.x % 16, tt = threadIdx.x / 16;
    float acc[RT][RC];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int c = 0; c < RC; ++c) acc[i][c] = 0.f;
#pragma unroll 4
    for (int a = 0; a < D; ++a) {
        float sv[RC];
        lds<RC>(sS + a * D + tc * RC, sv);
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const float qa = sQ[(tt * RT + i) * LDQ + a];
#pragma unroll
            for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(qa, sv[c], acc[i][c]);
        }
    }
    __syncthreads();
    T* Oh = out + bh * (long long)N * D;
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int row = row0 + tt * RT + i;
        if (row >= N) continue;
        const float den = normalize ? sDen[tt * RT + i] : 1.f;
#pragma unroll
        for (int c = 0; c < RC; ++c)
            Oh[(long long)row * D + tc * RC + c] = from_f32<T>(normalize ? acc[i][c] / den : acc[i][c]);
    }
}

// ---------------------------------------------------------------------------
// Chunked causal / prefix-mask outputs.
// ---------------------------------------------------------------------------
template <int D>
constexpr size_t chunked_smem() {
    return sizeof(float) * ((size_t)D * D + D + 3 * kC * (D + 4) + kC * (kC + 4) + kC) +
           2 * sizeof(int) * kC;
}

template <typename T, int D, bool GATHER>
__global__ void __launch_bounds__(kThreads)
chunked_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
               const float* __restrict__ prefix, int H, int N, int block_tokens, int nblk,
               const int32_t* __restrict__ perm, const int32_t* __restrict__ bin_start,
               const int32_t* __restrict__ msort, int nbins, int phi, int normalize,
               T* __restrict__ out) {
    constexpr int LD = D + 4, LDP = kC + 4;
    constexpr int R = D / 16;               // state-update block per thread (R x R)
    constexpr int RT = kC / 16, RC = D / 16;  // output block per thread (RT rows x RC cols)
    extern __shared__ __align__(16) float sm[];
    float* sS = sm;
    float* sz = sS + D * D;
    float* sQ = sz + D;
    float* sK = sQ + kC * LD;
    float* sV = sK + kC * LD;
    float* sP = sV + kC * LD;
    float* sDen = sP + kC * LDP;
    int* sRow = reinterpret_cast<int*>(sDen + kC);
    int* sLim = sRow + kC;

    const int blk = blockIdx.x;
    const long long bh = blockIdx.y;
    const int b = (int)(bh / H);
    const long long hoff = bh * (long long)N * D;
    const T* Qh = Q + hoff;
    const T* Kh = K + hoff;
    const T* Vh = V + hoff;
    T* Oh = out + hoff;

    pdl_wait();
    const float* pre = prefix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
    for (int e = threadIdx.x; e < D * D + D; e += kThreads) {
        if (e < D * D) sS[e] = pre[e];
        else sz[e - D * D] = pre[e];
    }
    const int nchunks = (N + kC - 1) / kC;
    const int c_begin = blk * (block_tokens / kC);
    int c_end = min(nchunks, c_begin + block_tokens / kC);
    if (GATHER && blk == nblk - 1) c_end = nbins;  // the last block also answers the all-keys bin

    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;
    const int tc = threadIdx.x % 16, tt = threadIdx.x / 16;

    for (int c = c_begin; c < c_end; ++c) {
        const int kvalid = c < nchunks ? min(kC, N - c * kC) : 0;
        __syncthreads();
        if (kvalid > 0) {
            tile_to_smem<T, D, LD>(sK, Kh + (long long)c * kC * D, kC, kvalid, true, phi);
            tile_to_smem<T, D, LD>(sV, Vh + (long long)c * kC * D, kC, kvalid, false, phi);
        } else {
            for (int e = threadIdx.x; e < kC * LD; e += kThreads) { sK[e] = 0.f; sV[e] = 0.f; }
        }
        int qbeg, qend;
        if (GATHER) {
            qbeg = bin_start[(size_t)b * (nbins + 1) + c];
            qend = bin_start[(size_t)b * (nbins + 1) + c + 1];
        } else {
            qbeg = 0;
            qend = kvalid;
        }
        for (int qt = qbeg; qt < qend; qt += kC) {
            const int nq = min(kC, qend - qt);
            __syncthreads();
            if (threadIdx.x < kC) {
                const int r = threadIdx.x;
                if (r < nq) {
                    if (GATHER) {
                        sRow[r] = perm[(size_t)b * N + qt + r];
                        sLim[r] = msort[(size_t)b * N + qt + r] - c * kC;  // in [-1, kvalid-1]
                    } else {
                        sRow[r] = c * kC + r;
                        sLim[r] = r;
                    }
                } else {
                    sRow[r] = -1;
                    sLim[r] = -1;
                }
            }
            __syncthreads();
            // phi(Q) rows of this tile
            {
                constexpr int EPV = Vec16<T>::N, VPR = D / EPV;
                for (int t = threadIdx.x; t < kC * VPR; t += kThreads) {
                    const int r = t / VPR, col = (t % VPR) * EPV;
                    float f[EPV];
                    const int i = sRow[r];
                    if (i >= 0) {
                        Vec16<T>::unpack(ldg_stream(Qh + (long long)i * D + col), f);
#pragma unroll
                        for (int e = 0; e < EPV; ++e) f[e] = phi_apply(f[e], phi);
                    } else {
#pragma unroll
                        for (int e = 0; e < EPV; ++e) f[e] = 0.f;
                    }
                    float4* o = reinterpret_cast<float4*>(sQ + r * LD + col);
#pragma unroll
                    for (int e = 0; e < EPV; e += 4) o[e / 4] = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
                }
            }
            __syncthreads();
            // P[i][j] = phi(q_i).phi(k_j) for visible j, else 0
            for (int idx = threadIdx.x; idx < kC * kC; idx += kThreads) {
                const int i = idx / kC, j = idx % kC;
                float p = 0.f;
                if (j <= sLim[i]) {
                    const float* qi = sQ + i * LD;
                    const float* kj = sK + j * LD;
#pragma unroll 8
                    for (int a = 0; a < D; ++a) p = fmaf(qi[a], kj[a], p);
                }
                sP[i * LDP + j] = p;
            }
            __syncthreads();
            if (normalize && threadIdx.x < kC) {
                const int i = threadIdx.x;
                float den = 0.f;
                for (int j = 0; j < kC; ++j) den += sP[i * LDP + j];
                float dz = 0.f;
                for (int a = 0; a < D; ++a) dz = fmaf(sQ[i * LD + a], sz[a], dz);
                sDen[i] = den + dz;
            }
            float acc[RT][RC];
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int cc = 0; cc < RC; ++cc) acc[i][cc] = 0.f;
            for (int j = 0; j < kC; ++j) {
                float vv[RC];
                lds<RC>(sV + j * LD + tc * RC, vv);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float pij = sP[(tt * RT + i) * LDP + j];
#pragma unroll
                    for (int cc = 0; cc < RC; ++cc) acc[i][cc] = fmaf(pij, vv[cc], acc[i][cc]);
                }
            }
#pragma unroll 4
            for (int a = 0; a < D; ++a) {
                float sv[RC];
                lds<RC>(sS + a * D + tc * RC, sv);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float qa = sQ[(tt * RT + i) * LD + a];
#pragma unroll
                    for (int cc = 0; cc < RC; ++cc) acc[i][cc] = fmaf(qa, sv[cc], acc[i][cc]);
                }
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const int r = tt * RT + i;
                const int row = sRow[r];
                if (row < 0) continue;
                const float den = normalize ? sDen[r] : 1.f;
#pragma unroll
                for (int cc = 0; cc < RC; ++cc)
                    Oh[(long long)row * D + tc * RC + cc] =
                        from_f32<T>(normalize ? acc[i][cc] / den : acc[i][cc]);
            }
        }
        // fold this chunk's keys into the running state
        if (kvalid > 0) {
            __syncthreads();
            float up[R][R];
            float zu[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                zu[r] = 0.f;
#pragma unroll
                for (int cc = 0; cc < R; ++cc) up[r][cc] = 0.f;
            }
            for (int j = 0; j < kC; ++j) {
                float a[R], bb[R];
                lds<R>(sK + j * LD + ta * R, a);
                lds<R>(sV + j * LD + tb * R, bb);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    zu[r] += a[r];
#pragma unroll
                    for (int cc = 0; cc < R; ++cc) up[r][cc] = fmaf(a[r], bb[cc], up[r][cc]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int cc = 0; cc < R; ++cc) sS[(ta * R + r) * D + tb * R + cc] += up[r][cc];
                if (tb == 0) sz[ta * R + r] += zu[r];
            }
        }
    }
}

template <typename T, int D>
cudaError_t launch_kv_partial(const Problem& p, const void* k, const void* v, int tps, int nsplit,
                              float* part, cudaStream_t st) {
    dim3 grid(nsplit, (unsigned)p.bh());
    return launch_pdl(kv_partial_kernel<T, D>, grid, dim3(kThreads), 0, st, static_cast<const T*>(k),
                      static_cast<const T*>(v), p.N, tps, nsplit, p.phi, part);
}

template <typename T, int D>
cudaError_t launch_readout(const Problem& p, const void* q, const float* S, const float* z,
                           void* out, cudaStream_t st) {
    constexpr size_t smem = readout_smem<D>();
    cudaError_t e = ensure_smem<readout_kernel<T, D>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.N + 63) / 64, (unsigned)p.bh());
    return launch_pdl(readout_kernel<T, D>, grid, dim3(kThreads), smem, st, static_cast<const T*>(q), S, z,
                      static_cast<T*>(out), p.N, p.phi, p.normalize);
}

template <typename T, int D>
cudaError_t launch_chunked(const Problem& p, const void* q, const void* k, const void* v,
                           const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                           const int32_t* bin_start, const int32_t* m, int nbins, void* out,
                           cudaStream_t st) {
    constexpr size_t smem = chunked_smem<D>();
    dim3 grid(nblk, (unsigned)p.bh());
    if (perm == nullptr) {
        cudaError_t e = ensure_smem<chunked_kernel<T, D, false>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(chunked_kernel<T, D, false>, grid, dim3(kThreads), smem, st,
                          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
                          prefix, p.H, p.N, block_tokens, nblk, (const int32_t*)nullptr,
                          (const int32_t*)nullptr, (const int32_t*)nullptr, 0, p.phi, p.normalize,
                          static_cast<T*>(out));
    } else {
        cudaError_t e = ensure_smem<chunked_kernel<T, D, true>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(chunked_kernel<T, D, true>, grid, dim3(kThreads), smem, st,
                          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
                          prefix, p.H, p.N, block_tokens, nblk, perm, bin_start, m, nbins, p.phi,
                          p.normalize, static_cast<T*>(out));
    }
}

}  // namespace

#define LA_DISPATCH(p, FN, ...)                                                              \
    do {                                                                                     \
        if ((p).dtype == DT_F32) {                                                           \
            switch ((p).d) {                                                                 \
                case 16: return FN<float, 16>(__VA_ARGS__);                                  \
                case 32: return FN<float, 32>(__VA_ARGS__);                                  \
                case 64: return FN<float, 64>(__VA_ARGS__);                                  \
                case 128: return FN<float, 128>(__VA_ARGS__);                                \
            }                                                                                \
        } else {                                                                             \
            switch ((p).d) {                                                                 \
                case 16: return FN<__nv_bfloat16, 16>(__VA_ARGS__);                          \
                case 32: return FN<__nv_bfloat16, 32>(__VA_ARGS__);                          \
                case 64: return FN<__nv_bfloat16, 64>(__VA_ARGS__);                          \
                case 128: return FN<__nv_bfloat16, 128>(__VA_ARGS__);                        \
            }                                                                                \
        }                                                                                    \
        return cudaErrorInvalidValue;                                                        \
    } while (0)

cudaError_t simt_kv_partial(const Problem& p, const void* k, const void* v, int tps, int nsplit,
                            float* part, cudaStream_t st) {
    LA_DISPATCH(p, launch_kv_partial, p, k, v, tps, nsplit, part, st);
}

cudaError_t simt_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                         cudaStream_t st) {
    LA_DISPATCH(p, launch_readout, p, q, S, z, out, st);
}

cudaError_t simt_chunked(const Problem& p, const void* q, const void* k, const void* v,
                         const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                         const int32_t* bin_start, const int32_t* m, int nbins, void* out,
                         cudaStream_t st) {
    LA_DISPATCH(p, launch_chunked, p, q, k, v, prefix, block_tokens, nblk, perm, bin_start, m,
                nbins, out, st);
}

cudaError_t state_reduce(const Problem& p, const float* part, int nsplit, float* S, float* z,
                         cudaStream_t st) {
    const int rec = p.d * p.d + p.d;
    dim3 grid((rec + 255) / 256, (unsigned)p.bh());
    return launch_pdl(state_reduce_kernel, grid, dim3(256), 0, st, part, nsplit, p.d, S, z);
}

cudaError_t state_exclusive_scan(const Problem& p, float* part, int nblk, float* S_total,
                                 float* z_total, cudaStream_t st, bool reverse) {
    const int rec4 = (p.d * p.d + p.d) / 4;
    dim3 grid((rec4 + 127) / 128, (unsigned)p.bh());
    return launch_pdl(state_scan_kernel, grid, dim3(128), 0, st, part, nblk, p.d, S_total, z_total,
                      reverse ? 1 : 0);
}

}  // namespace la
