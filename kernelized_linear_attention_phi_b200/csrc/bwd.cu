// Gradients of kernelized linear attention (non-causal and causal), on the
// CUDA cores with fp32 accumulation, for both element types and every d.
//
// The pages list a backward pass ("lineartile 1.0.1", "Project Structure":
// core/kernels/backward.py) without formulas; these are the derivatives of
// the forward definition. With a_i = phi(q_i), b_j = phi(k_j), the causal
// state S_i = sum_{j<=i} b_j v_j^T, z_i = sum_{j<=i} b_j (the non-causal
// form uses the totals for every i), num_i = a_i^T S_i, den_i = a_i . z_i,
// out_i = num_i / den_i, and g_i = dL/dout_i:
//   gn_i   = g_i / den_i,  gden_i = -(g_i . out_i) / den_i   (normalized;
//            unnormalized: gn_i = g_i, gden_i = 0)
//   dq_i   = phi'(q_i) * (S_i gn_i + z_i gden_i)
//   G_j    = sum_{i>=j} a_i gn_i^T,  h_j = sum_{i>=j} a_i gden_i
//   dk_j   = phi'(k_j) * (G_j v_j + h_j),   dv_j = G_j^T b_j
// So dq needs the prefix states the forward builds, and dk, dv need suffix
// states of (a, gn, gden): a forward sweep (bwd_q) computes out, den, gn,
// gden, dq and each block's own (G, h); a reverse exclusive scan over blocks
// gives the suffix states; a reverse sweep (bwd_kv) gives dk and dv. Within
// a chunk the intra-chunk terms use the masked C x C products
//   P_ij = a_i . b_j,  E_ij = gn_i . v_j + gden_i          (j <= i)
// (all ones above the diagonal for the non-causal form, where the chunk
// terms are folded into the totals instead and not formed).

#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "launch_util.h"

namespace la {
namespace {

constexpr int kThreads = 256;

template <int D>
struct BwCfg {
    static constexpr int C = D == 128 ? 32 : 64;  // tokens per chunk
    static constexpr int LD = D + 4;               // padded row of a [C x D] tile
    static constexpr int LDP = C + 4;              // padded row of a [C x C] tile
    static constexpr int R = D / 16;               // state block per thread (R x R)
    static constexpr int RT = C / 16, RC = D / 16;  // output block per thread (RT rows x RC cols)
    // S (or G) in both orientations, z (or h), four [C x D] tiles, one
    // [C x C] tile, two per-row vectors
    static constexpr size_t SMEM =
        sizeof(float) * (2 * (size_t)D * D + D + 4 * (size_t)C * LD + (size_t)C * LDP + 2 * C);
};

template <int R>
__device__ __forceinline__ void ldsv(const float* p, float* o) {
#pragma unroll
    for (int i = 0; i < R; i += 4) {
        if (R - i >= 4) {
            const float4 v = *reinterpret_cast<const float4*>(p + i);
            o[i] = v.x; o[i + 1] = v.y; o[i + 2] = v.z; o[i + 3] = v.w;
        } else {
#pragma unroll
            for (int e = i; e < R; ++e) o[e] = p[e];
        }
    }
}

// Loads a state (d x d matrix M[k][v] row-major, then a d vector) into M and
// its transpose in shared memory.
template <int D>
__device__ void load_state(const float* __restrict__ M, const float* __restrict__ vec, float* sM, float* sMT,
                           float* sv) {
    for (int e = threadIdx.x; e < D * D; e += kThreads) {
        const float x = M[e];
        sM[e] = x;
        sMT[(e % D) * D + e / D] = x;
    }
    for (int e = threadIdx.x; e < D; e += kThreads) sv[e] = vec[e];
}

// Masked C x C product out[i][j] = (A_i . B_j) (+ add) for visible (i, j),
// else 0; visible is j <= i (lower, add = add[i]) or j >= i (upper,
// add = add[j]). Register-tiled: thread (ti, tj) = (tid / 16, tid % 16)
// owns rows ti + 16 r and columns tj + 16 c and reads both operands as float4
// along d (rows interleaved so that neighbouring lanes read rows LD floats
// apart: LD / 4 = D / 4 + 1 is odd, so their 16-byte reads fall in distinct
// bank groups).
template <int D, bool LOWER>
__device__ void chunk_products(const float* sA_, const float* sB_, const float* add, float* sOut) {
    using CF = BwCfg<D>;
    constexpr int C = CF::C, LD = CF::LD, RB = C / 16;
    static_assert((LD / 4) % 2 == 1, "odd row stride in 16-byte units");
    const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
    float acc[RB][RB];
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int c = 0; c < RB; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int a = 0; a < D; a += 4) {
        float4 x[RB], y[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) x[r] = *reinterpret_cast<const float4*>(sA_ + (ti + 16 * r) * LD + a);
#pragma unroll
        for (int c = 0; c < RB; ++c) y[c] = *reinterpret_cast<const float4*>(sB_ + (tj + 16 * c) * LD + a);
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
            for (int c = 0; c < RB; ++c) {
                acc[r][c] = fmaf(x[r].x, y[c].x, acc[r][c]);
                acc[r][c] = fmaf(x[r].y, y[c].y, acc[r][c]);
                acc[r][c] = fmaf(x[r].z, y[c].z, acc[r][c]);
                acc[r][c] = fmaf(x[r].w, y[c].w, acc[r][c]);
            }
    }
#pragma unroll
    for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int c = 0; c < RB; ++c) {
            const int i = ti + 16 * r, j = tj + 16 * c;
            float p = 0.f;
            if (LOWER ? j <= i : j >= i) p = acc[r][c] + (add ? add[LOWER ? i : j] : 0.f);
            sOut[i * CF::LDP + j] = p;
        }
}

// ---------------------------------------------------------------------------
// Forward sweep: out, den, gn, gden, dq and the block's (G, h).
// ---------------------------------------------------------------------------
// Block blk of head bh covers tokens [blk * block_tokens, ...). Its state
// (S, z) is, causal: the exclusive prefix of the blocks before it (record
// bh * nblk + blk of Srec / zrec, stride rec); non-causal: the totals of the
// head (index bh).
template <typename T, int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads)
bwd_q_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
             const T* __restrict__ dO, const float* __restrict__ Sb, const float* __restrict__ zb,
             long long s_stride, long long z_stride, int N, int block_tokens, int nblk, int phi,
             int normalize, T* __restrict__ dQ, float* __restrict__ gn_out, float* __restrict__ gden_out,
             float* __restrict__ grec) {
    using CF = BwCfg<D>;
    constexpr int C = CF::C, LD = CF::LD, LDP = CF::LDP, R = CF::R, RT = CF::RT, RC = CF::RC;
    extern __shared__ __align__(16) float sm[];
    float* sS = sm;               // S [k][v]
    float* sST = sS + D * D;      // S^T [v][k]
    float* sz = sST + D * D;      // z [k]
    float* sA = sz + D;           // phi(q) [i][k]
    float* sB = sA + C * LD;      // phi(k) [j][k]      (causal)
    float* sV = sB + C * LD;      // v [j][v]           (causal)
    float* sG = sV + C * LD;      // dO, then gn [i][v]
    float* sP = sG + C * LD;      // P, then E [i][j]   (causal)
    float* sDen = sP + C * LDP;   // den [i]
    float* sGd = sDen + C;        // gden [i]

    const int blk = blockIdx.x;
    const long long bh = blockIdx.y;
    const long long hoff = bh * (long long)N * D;
    const int tt = threadIdx.x / 16, tc = threadIdx.x % 16;  // output rows / columns
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;  // state rows / columns
    pdl_wait();
    const long long si = CAUSAL ? bh * nblk + blk : bh;
    load_state<D>(Sb + si * s_stride, zb + si * z_stride, sS, sST, sz);

    float gacc[R][R], hacc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        hacc[r] = 0.f;
#pragma unroll
        for (int c = 0; c < R; ++c) gacc[r][c] = 0.f;
    }
    const int t_begin = blk * block_tokens, t_end = min(N, t_begin + block_tokens);
    for (int t0 = t_begin; t0 < t_end; t0 += C) {
        const int valid = min(C, t_end - t0);
        __syncthreads();
        tile_to_smem<T, D, LD>(sA, Q + hoff + (long long)t0 * D, C, valid, true, phi);
        tile_to_smem<T, D, LD>(sG, dO + hoff + (long long)t0 * D, C, valid, false, phi);
        if (CAUSAL) {
            tile_to_smem<T, D, LD>(sB, K + hoff + (long long)t0 * D, C, valid, true, phi);
            tile_to_smem<T, D, LD>(sV, V + hoff + (long long)t0 * D, C, valid, false, phi);
        }
        __syncthreads();
        if (CAUSAL) {
            chunk_products<D, true>(sA, sB, nullptr, sP);
            __syncthreads();
        }
        if (threadIdx.x < C) {
            const int i = threadIdx.x;
            float den = 0.f;
            if (CAUSAL)
                for (int j = 0; j <= i; ++j) den += sP[i * LDP + j];
            for (int a = 0; a < D; ++a) den = fmaf(sA[i * LD + a], sz[a], den);
            sDen[i] = den;
        }
        // num = a S (+ P V)
        float acc[RT][RC];
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int c = 0; c < RC; ++c) acc[i][c] = 0.f;
#pragma unroll 4
        for (int a = 0; a < D; ++a) {
            float sv[RC];
            ldsv<RC>(sS + a * D + tc * RC, sv);
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const float x = sA[(tt * RT + i) * LD + a];
#pragma unroll
                for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(x, sv[c], acc[i][c]);
            }
        }
        if (CAUSAL) {
            for (int j = 0; j < C; ++j) {
                float vv[RC];
                ldsv<RC>(sV + j * LD + tc * RC, vv);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float pij = sP[(tt * RT + i) * LDP + j];
#pragma unroll
                    for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(pij, vv[c], acc[i][c]);
                }
            }
        }
        __syncthreads();  // sDen written; every read of sP (P) done
        // gn, gden (rows past the end of the range contribute nothing)
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = tt * RT + i;
            const bool live = r < valid;
            const float den = sDen[r];
            const float inv = normalize && live ? 1.0f / den : 1.0f;
            float dot = 0.f;
#pragma unroll
            for (int c = 0; c < RC; ++c) {
                float* g = sG + r * LD + tc * RC + c;
                const float o = acc[i][c] * inv;
                dot = fmaf(*g, o, dot);
                const float gn = live ? *g * inv : 0.f;
                *g = gn;
                if (live) gn_out[hoff + (long long)(t0 + r) * D + tc * RC + c] = gn;
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (tc == 0) {
                const float gd = (normalize && live) ? -dot * inv : 0.f;
                sGd[r] = gd;
                if (live) gden_out[bh * (long long)N + t0 + r] = gd;
            }
        }
        __syncthreads();
        if (CAUSAL) {
            chunk_products<D, true>(sG, sV, sGd, sP);  // E_ij = gn_i . v_j + gden_i, j <= i
            __syncthreads();
        }
        // dA = S gn + z gden (+ E B); dq = phi'(q) * dA
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int c = 0; c < RC; ++c) acc[i][c] = sGd[tt * RT + i] * sz[tc * RC + c];
#pragma unroll 4
        for (int v = 0; v < D; ++v) {
            float sv[RC];
            ldsv<RC>(sST + v * D + tc * RC, sv);
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const float x = sG[(tt * RT + i) * LD + v];
#pragma unroll
                for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(x, sv[c], acc[i][c]);
            }
        }
        if (CAUSAL) {
            for (int j = 0; j < C; ++j) {
                float bb[RC];
                ldsv<RC>(sB + j * LD + tc * RC, bb);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float eij = sP[(tt * RT + i) * LDP + j];
#pragma unroll
                    for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(eij, bb[c], acc[i][c]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = tt * RT + i;
            if (r >= valid) continue;
            const long long row = hoff + (long long)(t0 + r) * D;
#pragma unroll
            for (int c = 0; c < RC; ++c) {
                const int col = tc * RC + c;
                dQ[row + col] = from_f32<T>(phi_grad(to_f32<T>(Q[row + col]), phi) * acc[i][c]);
            }
        }
        // the block's own (G, h): G[k][v] += a[i][k] gn[i][v], h[k] += a[i][k] gden[i]
        for (int i = 0; i < C; ++i) {
            float x[R], y[R];
            ldsv<R>(sA + i * LD + ta * R, x);
            ldsv<R>(sG + i * LD + tb * R, y);
            const float gd = sGd[i];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hacc[r] = fmaf(x[r], gd, hacc[r]);
#pragma unroll
                for (int c = 0; c < R; ++c) gacc[r][c] = fmaf(x[r], y[c], gacc[r][c]);
            }
        }
        if (CAUSAL) {
            __syncthreads();  // every read of S this chunk done
            // S += B^T V, z += sum B (this chunk's keys), in both orientations
            float up[R][R], zu[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                zu[r] = 0.f;
#pragma unroll
                for (int c = 0; c < R; ++c) up[r][c] = 0.f;
            }
            for (int j = 0; j < C; ++j) {
                float x[R], y[R];
                ldsv<R>(sB + j * LD + ta * R, x);
                ldsv<R>(sV + j * LD + tb * R, y);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    zu[r] += x[r];
#pragma unroll
                    for (int c = 0; c < R; ++c) up[r][c] = fmaf(x[r], y[c], up[r][c]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int c = 0; c < R; ++c) {
                    sS[(ta * R + r) * D + tb * R + c] += up[r][c];
                    sST[(tb * R + c) * D + ta * R + r] += up[r][c];
                }
                if (tb == 0) sz[ta * R + r] += zu[r];
            }
        }
    }
    float* g = grec + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int c = 0; c < R; ++c) g[(ta * R + r) * D + tb * R + c] = gacc[r][c];
        if (tb == 0) g[D * D + ta * R + r] = hacc[r];
    }
}

// ---------------------------------------------------------------------------
// Reverse sweep: dk and dv.
// ---------------------------------------------------------------------------
// Block blk starts from (G, h) of every query after it: causal, the suffix
// state of the blocks after blk (index bh * nblk + blk); non-causal, the
// totals of the head (index bh). Causal chunks are swept last to first,
// each adding its own queries to (G, h) after its keys are done.
template <typename T, int D, bool CAUSAL, typename TG = float>
__global__ void __launch_bounds__(kThreads)
bwd_kv_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
              const TG* __restrict__ gn_in, const float* __restrict__ gden_in,
              const float* __restrict__ Gb, const float* __restrict__ hb, long long g_stride,
              long long h_stride, int N, int block_tokens, int nblk, int phi, T* __restrict__ dK,
              T* __restrict__ dV) {
    using CF = BwCfg<D>;
    constexpr int C = CF::C, LD = CF::LD, LDP = CF::LDP, R = CF::R, RT = CF::RT, RC = CF::RC;
    extern __shared__ __align__(16) float sm[];
    float* sGm = sm;              // G [k][v]
    float* sGT = sGm + D * D;     // G^T [v][k]
    float* sh = sGT + D * D;      // h [k]
    float* sA = sh + D;           // phi(q) [i][k]      (causal)
    float* sN = sA + C * LD;      // gn [i][v]          (causal)
    float* sB = sN + C * LD;      // phi(k) [j][k]
    float* sV = sB + C * LD;      // v [j][v]
    float* sP = sV + C * LD;      // W^T, then E^T [j][i] (causal)
    float* sGd = sP + C * LDP;    // gden [i]           (causal)

    const int blk = blockIdx.x;
    const long long bh = blockIdx.y;
    const long long hoff = bh * (long long)N * D;
    const int tt = threadIdx.x / 16, tc = threadIdx.x % 16;
    const int ta = threadIdx.x / 16, tb = threadIdx.x % 16;
    pdl_wait();
    const long long si = CAUSAL ? bh * nblk + blk : bh;
    load_state<D>(Gb + si * g_stride, hb + si * h_stride, sGm, sGT, sh);

    const int t_begin = blk * block_tokens, t_end = min(N, t_begin + block_tokens);
    const int nch = (t_end - t_begin + C - 1) / C;
    for (int ci = 0; ci < nch; ++ci) {
        const int t0 = t_begin + (CAUSAL ? nch - 1 - ci : ci) * C;
        const int valid = min(C, t_end - t0);
        __syncthreads();
        tile_to_smem<T, D, LD>(sB, K + hoff + (long long)t0 * D, C, valid, true, phi);
        tile_to_smem<T, D, LD>(sV, V + hoff + (long long)t0 * D, C, valid, false, phi);
        if (CAUSAL) {
            tile_to_smem<T, D, LD>(sA, Q + hoff + (long long)t0 * D, C, valid, true, phi);
            tile_to_smem<TG, D, LD>(sN, gn_in + hoff + (long long)t0 * D, C, valid, false, phi);
            if (threadIdx.x < C)
                sGd[threadIdx.x] = threadIdx.x < valid ? gden_in[bh * (long long)N + t0 + threadIdx.x] : 0.f;
        }
        __syncthreads();
        if (CAUSAL) {
            chunk_products<D, false>(sB, sA, nullptr, sP);  // W^T[j][i] = b_j . a_i, i >= j
            __syncthreads();
        }
        // dv = G^T b (+ W^T gn)
        float acc[RT][RC];
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int c = 0; c < RC; ++c) acc[i][c] = 0.f;
#pragma unroll 4
        for (int k = 0; k < D; ++k) {
            float gv[RC];
            ldsv<RC>(sGm + k * D + tc * RC, gv);
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const float x = sB[(tt * RT + i) * LD + k];
#pragma unroll
                for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(x, gv[c], acc[i][c]);
            }
        }
        if (CAUSAL) {
            for (int i2 = 0; i2 < C; ++i2) {
                float nn[RC];
                ldsv<RC>(sN + i2 * LD + tc * RC, nn);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float w = sP[(tt * RT + i) * LDP + i2];
#pragma unroll
                    for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(w, nn[c], acc[i][c]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = tt * RT + i;
            if (r >= valid) continue;
            const long long row = hoff + (long long)(t0 + r) * D;
#pragma unroll
            for (int c = 0; c < RC; ++c) dV[row + tc * RC + c] = from_f32<T>(acc[i][c]);
        }
        if (CAUSAL) {
            __syncthreads();  // every read of W^T done
            chunk_products<D, false>(sV, sN, sGd, sP);  // E^T[j][i] = v_j . gn_i + gden_i, i >= j
            __syncthreads();
        }
        // dB = G v + h (+ E^T a); dk = phi'(k) * dB
#pragma unroll
        for (int i = 0; i < RT; ++i)
#pragma unroll
            for (int c = 0; c < RC; ++c) acc[i][c] = sh[tc * RC + c];
#pragma unroll 4
        for (int v = 0; v < D; ++v) {
            float gk[RC];
            ldsv<RC>(sGT + v * D + tc * RC, gk);
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                const float x = sV[(tt * RT + i) * LD + v];
#pragma unroll
                for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(x, gk[c], acc[i][c]);
            }
        }
        if (CAUSAL) {
            for (int i2 = 0; i2 < C; ++i2) {
                float aa[RC];
                ldsv<RC>(sA + i2 * LD + tc * RC, aa);
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const float e = sP[(tt * RT + i) * LDP + i2];
#pragma unroll
                    for (int c = 0; c < RC; ++c) acc[i][c] = fmaf(e, aa[c], acc[i][c]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const int r = tt * RT + i;
            if (r >= valid) continue;
            const long long row = hoff + (long long)(t0 + r) * D;
#pragma unroll
            for (int c = 0; c < RC; ++c) {
                const int col = tc * RC + c;
                dK[row + col] = from_f32<T>(phi_grad(to_f32<T>(K[row + col]), phi) * acc[i][c]);
            }
        }
        if (CAUSAL) {
            __syncthreads();  // every read of G this chunk done
            // G += A^T gn, h += A^T gden (this chunk's queries), both orientations
            float up[R][R], hu[R];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                hu[r] = 0.f;
#pragma unroll
                for (int c = 0; c < R; ++c) up[r][c] = 0.f;
            }
            for (int i2 = 0; i2 < C; ++i2) {
                float x[R], y[R];
                ldsv<R>(sA + i2 * LD + ta * R, x);
                ldsv<R>(sN + i2 * LD + tb * R, y);
                const float gd = sGd[i2];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    hu[r] = fmaf(x[r], gd, hu[r]);
#pragma unroll
                    for (int c = 0; c < R; ++c) up[r][c] = fmaf(x[r], y[c], up[r][c]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
#pragma unroll
                for (int c = 0; c < R; ++c) {
                    sGm[(ta * R + r) * D + tb * R + c] += up[r][c];
                    sGT[(tb * R + c) * D + ta * R + r] += up[r][c];
                }
                if (tb == 0) sh[ta * R + r] += hu[r];
            }
        }
    }
}

template <typename T, int D>
cudaError_t launch_bwd(const Problem& p, bool causal, const void* q, const void* k, const void* v,
                       const void* dout, const float* S, const float* z, long long s_stride, long long z_stride,
                       const float* G, const float* h, long long g_stride, long long h_stride, int block_tokens,
                       int nblk, void* dq, void* dk, void* dv, float* gn, float* gden, float* grec, bool q_pass,
                       bool gn16, cudaStream_t st) {
    using CF = BwCfg<D>;
    if (block_tokens % CF::C != 0) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)nblk, (unsigned)p.bh());
    const T* Q = static_cast<const T*>(q);
    const T* K = static_cast<const T*>(k);
    const T* V = static_cast<const T*>(v);
    if (q_pass) {
        auto kern = causal ? bwd_q_kernel<T, D, true> : bwd_q_kernel<T, D, false>;
        cudaError_t e = causal ? ensure_smem<bwd_q_kernel<T, D, true>>(CF::SMEM)
                               : ensure_smem<bwd_q_kernel<T, D, false>>(CF::SMEM);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, grid, dim3(kThreads), CF::SMEM, st, Q, K, V, static_cast<const T*>(dout), S, z,
                          s_stride, z_stride, p.N, block_tokens, nblk, p.phi, p.normalize, static_cast<T*>(dq), gn,
                          gden, grec);
    }
    if (gn16) {
        // gn in bf16 (from the tensor-core first sweep: causal, bf16, d = 64)
        if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 64) {
            if (!causal) return cudaErrorInvalidValue;
            cudaError_t e = ensure_smem<bwd_kv_kernel<T, D, true, __nv_bfloat16>>(CF::SMEM);
            if (e != cudaSuccess) return e;
            return launch_pdl(bwd_kv_kernel<T, D, true, __nv_bfloat16>, grid, dim3(kThreads), CF::SMEM, st, Q, K, V,
                              reinterpret_cast<const __nv_bfloat16*>(gn), static_cast<const float*>(gden), G, h,
                              g_stride, h_stride, p.N, block_tokens, nblk, p.phi, static_cast<T*>(dk),
                              static_cast<T*>(dv));
        }
        return cudaErrorInvalidValue;
    }
    auto kern = causal ? bwd_kv_kernel<T, D, true> : bwd_kv_kernel<T, D, false>;
    cudaError_t e = causal ? ensure_smem<bwd_kv_kernel<T, D, true>>(CF::SMEM)
                           : ensure_smem<bwd_kv_kernel<T, D, false>>(CF::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, grid, dim3(kThreads), CF::SMEM, st, Q, K, V, static_cast<const float*>(gn),
                      static_cast<const float*>(gden), G, h, g_stride, h_stride, p.N, block_tokens, nblk, p.phi,
                      static_cast<T*>(dk), static_cast<T*>(dv));
}

template <typename T>
cudaError_t bwd_dispatch(const Problem& p, bool causal, const void* q, const void* k, const void* v,
                         const void* dout, const float* S, const float* z, long long s_stride, long long z_stride,
                         const float* G, const float* h, long long g_stride, long long h_stride, int block_tokens,
                         int nblk, void* dq, void* dk, void* dv, float* gn, float* gden, float* grec, bool q_pass,
                         bool gn16, cudaStream_t st) {
#define LA_BW(D_)                                                                                             \
    return launch_bwd<T, D_>(p, causal, q, k, v, dout, S, z, s_stride, z_stride, G, h, g_stride, h_stride, \
                             block_tokens, nblk, dq, dk, dv, gn, gden, grec, q_pass, gn16, st)
    switch (p.d) {
        case 16: LA_BW(16);
        case 32: LA_BW(32);
        case 64: LA_BW(64);
        case 128: LA_BW(128);
    }
#undef LA_BW
    return cudaErrorInvalidValue;
}

}  // namespace

int bwd_chunk(const Problem& p) { return p.d == 128 ? BwCfg<128>::C : 64; }

cudaError_t bwd_q(const Problem& p, bool causal, const void* q, const void* k, const void* v, const void* dout,
                  const float* S, const float* z, long long s_stride, long long z_stride, int block_tokens,
                  int nblk, void* dq, float* gn, float* gden, float* grec, cudaStream_t st) {
    auto f = p.dtype == DT_F32 ? bwd_dispatch<float> : bwd_dispatch<__nv_bfloat16>;
    return f(p, causal, q, k, v, dout, S, z, s_stride, z_stride, nullptr, nullptr, 0, 0, block_tokens, nblk, dq,
             nullptr, nullptr, gn, gden, grec, true, false, st);
}

cudaError_t bwd_kv(const Problem& p, bool causal, const void* q, const void* k, const void* v, const void* gn,
                   const float* gden, const float* G, const float* h, long long g_stride, long long h_stride,
                   int block_tokens, int nblk, void* dk, void* dv, cudaStream_t st, bool gn_bf16) {
    auto f = p.dtype == DT_F32 ? bwd_dispatch<float> : bwd_dispatch<__nv_bfloat16>;
    return f(p, causal, q, k, v, nullptr, nullptr, nullptr, 0, 0, G, h, g_stride, h_stride, block_tokens, nblk,
             nullptr, dk, dv, static_cast<float*>(const_cast<void*>(gn)), const_cast<float*>(gden), nullptr, false,
             gn_bf16, st);
}

}  // namespace la
