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
#include "device.h"
#include "internal.h"
#include "launch_util.h"
#include "plan.h"

namespace la {
namespace {

constexpr int kThreads = 256;
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
template <int D>
struct KvRange {
    static constexpr int R = D / 16;                 // S rows and columns per thread
    static constexpr int TT = 2048 / D;              // tokens per tile (two tiles of K and V: 32 KB)
};

// Sums phi(K_t) (x) V_t and phi(K_t) over tokens [t0, t1) of one head, in
// token order, through two shared tiles of TT tokens (sK, sV: 2 x TT x D
// floats each). Thread (ta, tb) = (tid / 16, tid % 16) holds the R x R block
// of S at rows ta*R.., columns tb*R.., and z entries ta*R.. .
template <typename T, int D>
__device__ __forceinline__ void kv_range(const T* __restrict__ Kh, const T* __restrict__ Vh, int t0, int t1,
                                         int phi, float* sK, float* sV, float (&acc)[KvRange<D>::R][KvRange<D>::R],
                                         float (&zacc)[KvRange<D>::R]) {
    constexpr int R = KvRange<D>::R, kTT = KvRange<D>::TT;
    constexpr int EPV = Vec16<T>::N, VPR = D / EPV;
    constexpr int NV = kTT * VPR;                        // 16-byte vectors per tile and tensor
    constexpr int PER = (NV + kThreads - 1) / kThreads;  // of them per thread
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;

    // this thread's vectors of the tile at `base`, held in registers so that
    // the next tile's loads are in flight while the current one is summed
    uint4 rk[PER], rv[PER];
    auto fetch = [&](int base) {
        const int valid = min(kTT, t1 - base);
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int t = threadIdx.x + j * kThreads;
            const int r = t / VPR, col = (t % VPR) * EPV;
            const bool in = t < NV && r < valid;
            rk[j] = in ? ldg_stream(Kh + (size_t)(base + r) * D + col) : make_uint4(0, 0, 0, 0);
            rv[j] = in ? ldg_stream(Vh + (size_t)(base + r) * D + col) : make_uint4(0, 0, 0, 0);
        }
        return valid;
    };
    auto stage = [&](int buf, int valid) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int t = threadIdx.x + j * kThreads;
            if (t >= NV) continue;
            const int r = t / VPR, col = (t % VPR) * EPV;
            float fk[EPV], fv[EPV];
            Vec16<T>::unpack(rk[j], fk);
            Vec16<T>::unpack(rv[j], fv);
#pragma unroll
            for (int e = 0; e < EPV; ++e) fk[e] = r < valid ? phi_apply(fk[e], phi) : 0.f;
            float* dk = sK + buf * kTT * D + r * D + col;
            float* dv = sV + buf * kTT * D + r * D + col;
#pragma unroll
            for (int e = 0; e < EPV; e += 4) {
                *reinterpret_cast<float4*>(dk + e) = make_float4(fk[e], fk[e + 1], fk[e + 2], fk[e + 3]);
                *reinterpret_cast<float4*>(dv + e) = make_float4(fv[e], fv[e + 1], fv[e + 2], fv[e + 3]);
            }
        }
    };

#pragma unroll
    for (int r = 0; r < R; ++r) {
        zacc[r] = 0.f;
#pragma unroll
        for (int c = 0; c < R; ++c) acc[r][c] = 0.f;
    }
    int buf = 0;
    if (t0 < t1) stage(0, fetch(t0));
    __syncthreads();
    for (int base = t0; base < t1; base += kTT) {
        const bool more = base + kTT < t1;
        const int nvalid = more ? fetch(base + kTT) : 0;
#pragma unroll 4
        for (int t = 0; t < kTT; ++t) {
            float a[R], bb[R];
            lds<R>(sK + buf * kTT * D + t * D + ta * R, a);
            lds<R>(sV + buf * kTT * D + t * D + tb * R, bb);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                zacc[r] += a[r];
#pragma unroll
                for (int c = 0; c < R; ++c) acc[r][c] = fmaf(a[r], bb[c], acc[r][c]);
            }
        }
        if (more) stage(buf ^ 1, nvalid);
        __syncthreads();
        buf ^= 1;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
kv_partial_kernel(const T* __restrict__ K, const T* __restrict__ V, int N, int tps, int nsplit,
                  int phi, float* __restrict__ part) {
    constexpr int R = KvRange<D>::R, kTT = KvRange<D>::TT;
    __shared__ __align__(16) float sK[2 * kTT * D];
    __shared__ __align__(16) float sV[2 * kTT * D];
    const int s = blockIdx.x;
    const long long bh = blockIdx.y;
    const int t0 = s * tps;
    const int t1 = min(N, t0 + tps);
    pdl_wait();
    float acc[R][R], zacc[R];
    kv_range<T, D>(K + bh * (long long)N * D, V + bh * (long long)N * D, t0, t1, phi, sK, sV, acc, zacc);
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;
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
template <int D, int TQ = 64>
constexpr size_t readout_smem() {
    return sizeof(float) * ((size_t)D * D + D + TQ * (D + 4) + TQ);
}

// Outputs of query rows row0 .. row0 + TQ - 1 of one head from S, z in
// shared memory (sS [D x D], sz [D]); sQ and sDen are the tile's scratch.
template <typename T, int D, int TQ = 64>
__device__ __forceinline__ void readout_rows(const T* __restrict__ Qh, T* __restrict__ Oh, int row0, int N,
                                             int phi, int normalize, const float* sS, const float* sz,
                                             float* sQ, float* sDen) {
    constexpr int LDQ = D + 4, RC = D / 16, RT = TQ / 16;
    static_assert(TQ <= kThreads, "one thread per row for the denominators");
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

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
readout_kernel(const T* __restrict__ Q, const float* __restrict__ S, const float* __restrict__ z,
               T* __restrict__ out, int N, int phi, int normalize) {
    constexpr int TQ = 64, LDQ = D + 4;
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
    readout_rows<T, D>(Q + bh * (long long)N * D, out + bh * (long long)N * D, tile * TQ, N, phi, normalize,
                       sS, sz, sQ, sDen);
}

// ---------------------------------------------------------------------------
// Small non-causal problems in one launch: one CTA per head forms S and z
// over all of the head's keys (kv_range with a single split), keeps them in
// shared memory (and writes them out when asked), then reads out all of the
// head's queries 64 rows at a time (readout_rows). Replaces the three
// dependent launches (partials, reduction, readout) where a head is short.
// ---------------------------------------------------------------------------
// query rows per readout pass of the one-launch kernel: all of a 256-token
// head at d = 16 (16 rows per thread), half of it at d = 32
template <int D>
struct SmallTQ {
    static constexpr int value = D <= 16 ? 256 : 128;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
noncausal_small_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                       T* __restrict__ out, float* __restrict__ S_out, float* __restrict__ z_out, int N,
                       int phi, int normalize) {
    constexpr int R = KvRange<D>::R, kTT = KvRange<D>::TT, TQ = SmallTQ<D>::value, LDQ = D + 4;
    extern __shared__ __align__(16) float sm[];
    float* sK = sm;                // two K tiles, then two V tiles
    float* sV = sK + 2 * kTT * D;
    float* sS = sV + 2 * kTT * D;
    float* sz = sS + D * D;
    float* sQ = sz + D;
    float* sDen = sQ + TQ * LDQ;
    const long long bh = blockIdx.x;
    pdl_wait();
    const T* Qh = Q + bh * (long long)N * D;
    // the head's queries (at most 32 KB) move towards L2 while S and z form
    for (long long off = threadIdx.x * 128LL; off < (long long)N * D * (long long)sizeof(T); off += kThreads * 128LL)
        prefetch_l2(reinterpret_cast<const char*>(Qh) + off);
    float acc[R][R], zacc[R];
    kv_range<T, D>(K + bh * (long long)N * D, V + bh * (long long)N * D, 0, N, phi, sK, sV, acc, zacc);
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int c = 0; c < R; ++c) sS[(ta * R + r) * D + tb * R + c] = acc[r][c];
        if (tb == 0) sz[ta * R + r] = zacc[r];
        if (S_out != nullptr) {
#pragma unroll
            for (int c = 0; c < R; ++c) S_out[(size_t)bh * D * D + (ta * R + r) * D + tb * R + c] = acc[r][c];
            if (tb == 0) z_out[(size_t)bh * D + ta * R + r] = zacc[r];
        }
    }
    T* Oh = out + bh * (long long)N * D;
    for (int row0 = 0; row0 < N; row0 += TQ) {
        __syncthreads();  // S, z written; the previous tile's sQ and sDen read
        readout_rows<T, D, TQ>(Qh, Oh, row0, N, phi, normalize, sS, sz, sQ, sDen);
    }
}

// ---------------------------------------------------------------------------
// Chunked causal / prefix-mask outputs.
//
// Every product is a small matrix product over shared-memory tiles stored
// with the output's row index contiguous along the contraction ("k-major"),
// so that a thread reads four consecutive rows (or columns) with one 16-byte
// load per contraction step and accumulates a 4 x RC block in registers:
//   P^T  = (phi(Q)^T)^T (phi(K)^T)      queries x keys, masked, stored [key][query]
//   O    = phi(Q) S + P V               queries x d_v
//   S   += phi(K)^T V,  z += phi(K)^T 1
// ---------------------------------------------------------------------------
template <int D>
struct ChCfg {
    static constexpr int C = kC;
    static constexpr int LC = C + 4;        // row length of the [D][C] and [C][C] tiles
    static constexpr int LDD = D + 4;       // row length of the [C][D] and [D][D] tiles
    static constexpr int RC = D / 16;       // output columns per thread (O, S)
    static constexpr int OFF_S = 0, OFF_Z = OFF_S + D * LDD, OFF_QT = OFF_Z + D, OFF_KT = OFF_QT + D * LC,
                         OFF_KN = OFF_KT + D * LC, OFF_VN = OFF_KN + C * LDD, OFF_PT = OFF_VN + C * LDD,
                         OFF_DEN = OFF_PT + C * LC, FLOATS = OFF_DEN + C;
    static constexpr size_t SMEM = sizeof(float) * (size_t)FLOATS + 2 * sizeof(int) * C;
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int D>
constexpr size_t chunked_smem() {
    return ChCfg<D>::SMEM;
}

// acc[r][c] += sum_k A[k][i0 + r] * B[k][j0 + c], r < RI, c < RJ; A and B
// k-major with row lengths lda, ldb (multiples of 4 floats).
template <int RI, int RJ>
__device__ __forceinline__ void kmajor_acc(float (&acc)[RI][RJ], const float* A, int lda, int i0, const float* B,
                                           int ldb, int j0, int K) {
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        float a[RI], b[RJ];
        lds<RI>(A + k * lda + i0, a);
        lds<RJ>(B + k * ldb + j0, b);
#pragma unroll
        for (int r = 0; r < RI; ++r)
#pragma unroll
            for (int c = 0; c < RJ; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
    }
}

// Rows of a [C x D] input tile into shared memory, phi applied when asked:
// transposed (dstT[col][row], row length LC) and/or natural (dstN[row][col],
// row length LDD). Row r of the tile is src row `rowidx(r)`; a negative
// index, or r >= valid, gives a zero row.
template <typename T, int D, typename RowIdx>
__device__ __forceinline__ void load_rows(const T* src, int valid, RowIdx rowidx, bool apply_phi, int phi,
                                          float* dstT, float* dstN) {
    using CF = ChCfg<D>;
    constexpr int EPV = Vec16<T>::N, VPR = D / EPV;
    for (int t = threadIdx.x; t < CF::C * VPR; t += kThreads) {
        const int r = t / VPR, col = (t % VPR) * EPV;
        const int row = r < valid ? rowidx(r) : -1;
        float f[EPV];
        if (row >= 0) {
            Vec16<T>::unpack(ldg_stream(src + (size_t)row * D + col), f);
            if (apply_phi) {
#pragma unroll
                for (int e = 0; e < EPV; ++e) f[e] = phi_apply(f[e], phi);
            }
        } else {
#pragma unroll
            for (int e = 0; e < EPV; ++e) f[e] = 0.f;
        }
        if (dstT) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) dstT[(col + e) * CF::LC + r] = f[e];
        }
        if (dstN) {
#pragma unroll
            for (int e = 0; e < EPV; e += 4)
                *reinterpret_cast<float4*>(dstN + r * CF::LDD + col + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
        }
    }
}

template <typename T, int D, bool GATHER>
__global__ void __launch_bounds__(kThreads)
chunked_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
               const float* __restrict__ prefix, int H, int N, int block_tokens, int nblk,
               const int32_t* __restrict__ perm, const int32_t* __restrict__ bin_start,
               const int32_t* __restrict__ msort, int nbins, int phi, int normalize,
               T* __restrict__ out) {
    using CF = ChCfg<D>;
    constexpr int C = CF::C, LC = CF::LC, LDD = CF::LDD, RC = CF::RC;
    extern __shared__ __align__(16) float sm[];
    float* sS = sm + CF::OFF_S;
    float* sz = sm + CF::OFF_Z;
    float* sQT = sm + CF::OFF_QT;
    float* sKT = sm + CF::OFF_KT;
    float* sKn = sm + CF::OFF_KN;
    float* sVn = sm + CF::OFF_VN;
    float* sPT = sm + CF::OFF_PT;
    float* sDen = sm + CF::OFF_DEN;
    int* sRow = reinterpret_cast<int*>(sm + CF::FLOATS);
    int* sLim = sRow + C;

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
    for (int e = threadIdx.x; e < D * D; e += kThreads) sS[(e / D) * LDD + e % D] = pre[e];
    for (int e = threadIdx.x; e < D; e += kThreads) sz[e] = pre[D * D + e];
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    int c_end = min(nchunks, c_begin + block_tokens / C);
    if (GATHER && blk == nblk - 1) c_end = nbins;  // the last block also answers the all-keys bin

    // output blocks: rows 4*ti .. 4*ti + 3 (queries), columns RC*tb .. (of d_v)
    // P blocks: rows 4*ti, keys 4*tj .. 4*tj + 3; state blocks: rows RC*ti (d_k)
    const int ti = threadIdx.x % 16, tj = threadIdx.x / 16;

    for (int c = c_begin; c < c_end; ++c) {
        const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
        __syncthreads();  // the previous chunk's tiles are no longer read
        load_rows<T, D>(Kh + (long long)c * C * D, kvalid, [](int r) { return r; }, true, phi, sKT, sKn);
        load_rows<T, D>(Vh + (long long)c * C * D, kvalid, [](int r) { return r; }, false, phi, nullptr, sVn);
        int qbeg, qend;
        if (GATHER) {
            qbeg = bin_start[(size_t)b * (nbins + 1) + c];
            qend = bin_start[(size_t)b * (nbins + 1) + c + 1];
        } else {
            qbeg = 0;
            qend = kvalid;
        }
        for (int qt = qbeg; qt < qend; qt += C) {
            const int nq = min(C, qend - qt);
            __syncthreads();  // the previous tile's queries, P and row table are no longer read
            if (threadIdx.x < C) {
                const int r = threadIdx.x;
                if (r < nq) {
                    sRow[r] = GATHER ? perm[(size_t)b * N + qt + r] : c * C + r;
                    sLim[r] = GATHER ? msort[(size_t)b * N + qt + r] - c * C : r;  // keys 0..lim visible
                } else {
                    sRow[r] = -1;
                    sLim[r] = -1;
                }
            }
            __syncthreads();
            load_rows<T, D>(Qh, nq, [&](int r) { return sRow[r]; }, true, phi, sQT, nullptr);
            __syncthreads();
            // P^T: queries x keys, masked
            {
                float p[4][4] = {};
                kmajor_acc<4, 4>(p, sQT, LC, 4 * ti, sKT, LC, 4 * tj, D);
                int lim[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) lim[r] = sLim[4 * ti + r];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int j = 4 * tj + cc;
                    *reinterpret_cast<float4*>(sPT + j * LC + 4 * ti) =
                        make_float4(j <= lim[0] ? p[0][cc] : 0.f, j <= lim[1] ? p[1][cc] : 0.f,
                                    j <= lim[2] ? p[2][cc] : 0.f, j <= lim[3] ? p[3][cc] : 0.f);
                }
            }
            __syncthreads();
            // denominators: the row sums of P~ in key order, then phi(q).z
            if (normalize && threadIdx.x < C) {
                const int i = threadIdx.x;
                float den = 0.f;
                for (int j = 0; j < C; ++j) den += sPT[j * LC + i];
                float dz = 0.f;
                for (int a = 0; a < D; ++a) dz = fmaf(sQT[a * LC + i], sz[a], dz);
                sDen[i] = den + dz;
            }
            // O = phi(Q) S + P V
            float o[4][RC] = {};
            kmajor_acc<4, RC>(o, sQT, LC, 4 * ti, sS, LDD, RC * tj, D);
            kmajor_acc<4, RC>(o, sPT, LC, 4 * ti, sVn, LDD, RC * tj, C);
            __syncthreads();  // sDen
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = 4 * ti + r;
                const int row = sRow[i];
                if (row < 0) continue;
                const float inv = normalize ? 1.f / sDen[i] : 1.f;
                float f[RC];
#pragma unroll
                for (int cc = 0; cc < RC; ++cc) f[cc] = o[r][cc] * inv;
                T* dst = Oh + (long long)row * D + RC * tj;
#pragma unroll
                for (int cc = 0; cc < RC; ++cc) dst[cc] = from_f32<T>(f[cc]);
            }
        }
        // fold this chunk's keys into the running state
        if (kvalid > 0) {
            __syncthreads();
            float up[RC][RC] = {};
            kmajor_acc<RC, RC>(up, sKn, LDD, RC * ti, sVn, LDD, RC * tj, C);
            float zu = 0.f;
            if (threadIdx.x < D)
                for (int j = 0; j < C; ++j) zu += sKn[j * LDD + threadIdx.x];
            __syncthreads();  // every read of the old state is done
#pragma unroll
            for (int r = 0; r < RC; ++r)
#pragma unroll
                for (int cc = 0; cc < RC; ++cc) sS[(RC * ti + r) * LDD + RC * tj + cc] += up[r][cc];
            if (threadIdx.x < D) sz[threadIdx.x] += zu;
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
cudaError_t launch_noncausal_small(const Problem& p, const void* q, const void* k, const void* v, void* out,
                                   float* S_out, float* z_out, cudaStream_t st) {
    if constexpr (D > 32) {
        return cudaErrorInvalidValue;
    } else {
        constexpr size_t smem = 4 * sizeof(float) * KvRange<D>::TT * D + readout_smem<D, SmallTQ<D>::value>();
        cudaError_t e = ensure_smem<noncausal_small_kernel<T, D>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(noncausal_small_kernel<T, D>, dim3((unsigned)p.bh()), dim3(kThreads), smem, st,
                          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
                          static_cast<T*>(out), S_out, z_out, p.N, p.phi, p.normalize);
    }
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

bool simt_noncausal_small_supported(const Problem& p) { return plan::small_noncausal(p, device_sms()); }

cudaError_t simt_noncausal_small(const Problem& p, const void* q, const void* k, const void* v, void* out,
                                 float* S_out, float* z_out, cudaStream_t st) {
    if (!simt_noncausal_small_supported(p)) return cudaErrorInvalidValue;
    LA_DISPATCH(p, launch_noncausal_small, p, q, k, v, out, S_out, z_out, st);
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
