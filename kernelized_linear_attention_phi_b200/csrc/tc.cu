// Tensor-core kernels (tcgen05 + TMEM + TMA) for bf16 inputs, d = 64 or 128.
//
// KV summary ("nx_f32_linear_attention.nx source", KV-summary loop):
//   S = phi(K)^T V over a token range, as MMAs with M = d_k, N = d_v and the
//   tokens as the contraction dimension. TMA stages 128-token K and V tiles;
//   four warps prepare K in shared memory (and sum z = sum phi(K) in fp32 on
//   the way); one thread issues tcgen05.mma with S accumulating in TMEM.
//   For phi = relu+1 the operand is relu(K), which is exact in bf16, and the
//   "+1" part is added as 1 (x) colsum(V): a second MMA against an all-ones
//   operand gives colsum(V). So S carries no rounding of phi(K) to bf16.
// Readout (nx source, per-query loop):
//   out = phi(Q) S / (phi(Q) . z) for 128-token tiles: MMA with M = tokens,
//   N = d_v, K = d_k against S in shared memory (bf16), and a second
//   N = 16 MMA against z for the denominator; the division and the bf16
//   store run in the TMEM epilogue.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues MMAs, warps 2-5 transform tiles (phi) and run epilogues.

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kTcThreads = 192;
constexpr int kTile = 128;  // tokens per TMA tile

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void unpack8(const uint4& w, float* f) { Vec16<__nv_bfloat16>::unpack(w, f); }
__device__ __forceinline__ uint4 pack8(const float* f) { return Vec16<__nv_bfloat16>::pack(f); }

// ---------------------------------------------------------------------------
// Partial KV summaries
// ---------------------------------------------------------------------------
template <int D>
struct KvCfg {
    static constexpr int NB = D / 64;                 // 64-column boxes per tile
    static constexpr int TILE = kTile * D * 2;        // bytes of a K or V tile
    static constexpr int STAGES = D == 64 ? 4 : 3;
    static constexpr int ONES = kTile * 128;           // all-ones MN-major operand (M = 64)
    static constexpr int ZRED = 128 * NB * 8 * 4;     // z partial sums
    static constexpr int BARS = 3 * STAGES + 1;
    static constexpr uint32_t TMEM_COLS = D == 64 ? 128 : 256;  // S, then the colsum block
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * 2 * TILE + ONES + ZRED + 8 * BARS + 16;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_kv_partial_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                     int N, int tps, int nsplit, int phi, float* __restrict__ part,
                     uint32_t* __restrict__ err) {
    using C = KvCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* ones = tiles + C::STAGES * 2 * C::TILE;
    float* zred = reinterpret_cast<float*>(ones + C::ONES);
    uint64_t* full = reinterpret_cast<uint64_t*>(zred + 128 * C::NB * 8);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* done = empty + C::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int split = blockIdx.x;
    const int bh = blockIdx.y;
    const int t0 = split * tps;
    const int t1 = min(N, t0 + tps);
    const int ntiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (threadIdx.x == 0) {
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
    }
    const bool relu = phi == PHI_RELU1;
    if (relu) {
        const uint4 one8 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (int c = threadIdx.x; c < C::ONES / 16; c += kTcThreads) reinterpret_cast<uint4*>(ones)[c] = one8;
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, 2 * C::TILE);
                uint8_t* kt = tiles + s * 2 * C::TILE;
                const int row = t0 + it * kTile;
#pragma unroll
                for (int b = 0; b < C::NB; ++b) {
                    tma_load_3d(kt + b * kTile * 128, &mK, full + s, b * 64, row, bh);
                    tma_load_3d(kt + C::TILE + b * kTile * 128, &mV, full + s, b * 64, row, bh);
                }
                issued[s] = u + 1;
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(D, D, true, true);
            constexpr uint32_t idesc_ones = idesc_bf16(64, D, true, true);
            const uint32_t ob = smem_u32(ones);
            for (int it = 0; it < ntiles; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (!mbar_wait(tdone + s, u & 1, err)) break;
                tc_fence_after();
                const uint32_t kt = smem_u32(tiles + s * 2 * C::TILE);
                const uint32_t vt = kt + C::TILE;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t a = sdesc(kt + kk * 2048, kTile * 128, 1024);
                    const uint64_t b = sdesc(vt + kk * 2048, kTile * 128, 1024);
                    mma_bf16(tmem, a, b, idesc, (it > 0 || kk > 0) ? 1u : 0u);
                    if (relu)  // every row of this block is colsum(V)
                        mma_bf16(tmem + D, sdesc(ob + kk * 2048, kTile * 128, 1024), b, idesc_ones,
                                 (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(empty + s);
            }
            mma_commit(done);
        }
    } else {
        const int et = threadIdx.x - 64;  // 0..127
        float zacc[C::NB][8];
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
#pragma unroll
            for (int e = 0; e < 8; ++e) zacc[b][e] = 0.f;
        bool ok = true;
        for (int it = 0; it < ntiles && ok; ++it) {
            const int s = it % C::STAGES, u = it / C::STAGES;
            ok = mbar_wait(full + s, u & 1, err);
            if (!ok) break;
            const int valid = min(kTile, t1 - (t0 + it * kTile));
            uint4* kt = reinterpret_cast<uint4*>(tiles + s * 2 * C::TILE);
#pragma unroll
            for (int i = 0; i < C::NB * 8; ++i) {
                const int p = et + 128 * i;   // 16-byte chunk index
                const int b = i / 8;          // box
                const int r = (p & 1023) >> 3;  // token row within the tile
                float f[8];
                unpack8(kt[p], f);
                if (r < valid) {
                    // operand: relu(k) for phi = relu+1 (exact in bf16), k for identity
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float ph = phi_apply(f[e], phi);
                        zacc[b][e] += ph;
                        f[e] = relu ? ph - 1.0f : ph;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = 0.f;
                }
                kt[p] = pack8(f);
            }
            fence_async_smem();
            mbar_arrive(tdone + s);
        }
        // z: the 16 threads sharing a column group hold its partial sums
#pragma unroll
        for (int b = 0; b < C::NB; ++b)
#pragma unroll
            for (int e = 0; e < 8; ++e) zred[et * C::NB * 8 + b * 8 + e] = zacc[b][e];
        named_bar(1, 128);
        float* rec = part + ((size_t)bh * nsplit + split) * (size_t)(D * D + D);
        if (et < D) {
            const int b = et / 64, g = (et % 64) / 8, e = et % 8;
            float zs = 0.f;
            for (int t = 0; t < 128; ++t)
                if ((((t & 7) ^ ((t >> 3) & 7))) == g) zs += zred[t * C::NB * 8 + b * 8 + e];
            rec[D * D + et] = zs;
        }
        // S from TMEM: lane = row of S (d_k index), columns = d_v
        const int sp = warp & 3;
        const bool have = ntiles > 0 && ok && mbar_wait(done, 0, err);
        tc_fence_after();
        constexpr int ROWS_PER_WARP = D == 128 ? 32 : 16;
        const int a = sp * ROWS_PER_WARP + lane;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + (static_cast<uint32_t>(sp * 32) << 16) + c0, r);
            if (relu) {
                // lanes 0..15 of each sub-partition hold a row of the M = 64
                // colsum block; every such row equals colsum(V)
                uint32_t c[16];
                tmem_ld16(tmem + (static_cast<uint32_t>(sp * 32) << 16) + D + c0, c);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    r[e] = __float_as_uint(__uint_as_float(r[e]) +
                                           __uint_as_float(__shfl_sync(0xffffffffu, c[e], lane & 15)));
            }
            tmem_ld_wait();
            if (lane < ROWS_PER_WARP) {
                float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    o[q] = have ? make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Readout
// ---------------------------------------------------------------------------
template <int D>
struct RoCfg {
    static constexpr int NB = D / 64;
    static constexpr int TILE = kTile * D * 2;         // Q tile bytes
    static constexpr int STAGES = D == 64 ? 4 : 3;
    static constexpr int BS = D * D * 2;               // S, MN-major bf16
    static constexpr int BZ = 16 * D * 2;              // z row + 15 zero rows, K-major
    static constexpr int ACC = D + 16;                 // accumulator columns per buffer
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256 : 512;
    static constexpr int BARS = 3 * STAGES + 4;
    // d = 64 pads shared memory so that at most two CTAs share an SM (their
    // TMEM allocations then always fit side by side).
    static constexpr size_t SMEM_USED = 1024 + (size_t)STAGES * TILE + BS + BZ + 8 * BARS + 16;
    static constexpr size_t SMEM = D == 64 ? (SMEM_USED > 80 * 1024 ? SMEM_USED : 80 * 1024) : SMEM_USED;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_readout_kernel(const __grid_constant__ CUtensorMap mQ, const float* __restrict__ S,
                  const float* __restrict__ z, __nv_bfloat16* __restrict__ out, int N, int phi,
                  int normalize, uint32_t* __restrict__ err) {
    using C = RoCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* bS = tiles + C::STAGES * C::TILE;
    uint8_t* bZ = bS + C::BS;
    uint64_t* full = reinterpret_cast<uint64_t*>(bZ + C::BZ);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* acc_full = empty + C::STAGES;   // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int bh = blockIdx.y;
    const int ntiles_head = (N + kTile - 1) / kTile;
    const int my_tiles = blockIdx.x < ntiles_head ? (ntiles_head - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full + a, 1);
            mbar_init(acc_empty + a, 128);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (threadIdx.x == 0) tma_prefetch_map(&mQ);

    // S -> bf16, MN-major (rows = d_k index a, 64-wide d_v atoms LBO = D*128 apart)
    const float* Sh = S + (size_t)bh * D * D;
    for (int c = threadIdx.x; c < D * D / 8; c += kTcThreads) {
        const int a = c / (D / 8), col = (c % (D / 8)) * 8;
        const float4 x0 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[0];
        const float4 x1 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[1];
        const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        *reinterpret_cast<uint4*>(bS + (col / 64) * (D * 128) + sw128_off(a, col % 64)) = pack8(f);
    }
    // z -> row 0 of a 16-row K-major operand (rows 1..15 zero)
    for (int c = threadIdx.x; c < 16 * D / 8; c += kTcThreads) {
        const int n = c / (D / 8), col = (c % (D / 8)) * 8;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = n == 0 ? z[(size_t)bh * D + col + e] : 0.f;
        *reinterpret_cast<uint4*>(bZ + (col / 64) * (16 * 128) + sw128_off(n, col % 64)) = pack8(f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int it = 0; it < my_tiles; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, C::TILE);
                const int tile = blockIdx.x + it * gridDim.x;
#pragma unroll
                for (int b = 0; b < C::NB; ++b)
                    tma_load_3d(tiles + s * C::TILE + b * kTile * 128, &mQ, full + s, b * 64,
                                tile * kTile, bh);
                issued[s] = u + 1;
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, D, false, true);
            constexpr uint32_t id_z = idesc_bf16(128, 16, false, false);
            const uint32_t sb = smem_u32(bS), zb = smem_u32(bZ);
            for (int it = 0; it < my_tiles; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                const int ab = it & 1, ua = it >> 1;
                if (!mbar_wait(tdone + s, u & 1, err)) break;
                if (ua > 0 && !mbar_wait(acc_empty + ab, (ua - 1) & 1, err)) break;
                tc_fence_after();
                const uint32_t qt = smem_u32(tiles + s * C::TILE);
                const uint32_t acc = tmem + ab * C::ACC;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = sdesc(qt + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024);
                    mma_bf16(acc, a, sdesc(sb + kk * 2048, D * 128, 1024), id_s, kk > 0 ? 1u : 0u);
                    if (normalize)
                        mma_bf16(acc + D, a, sdesc(zb + (kk / 4) * (16 * 128) + (kk % 4) * 32, 16, 1024),
                                 id_z, kk > 0 ? 1u : 0u);
                }
                mma_commit(empty + s);
                mma_commit(acc_full + ab);
            }
        }
    } else {
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const bool relu = phi == PHI_RELU1;
        bool ok = true;
        auto transform = [&](int it) {
            const int s = it % C::STAGES, u = it / C::STAGES;
            ok = ok && mbar_wait(full + s, u & 1, err);
            if (!ok) return;
            if (relu) {
                uint4* qt = reinterpret_cast<uint4*>(tiles + s * C::TILE);
#pragma unroll
                for (int i = 0; i < C::NB * 8; ++i) {
                    float f[8];
                    unpack8(qt[et + 128 * i], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = phi_relu1(f[e]);
                    qt[et + 128 * i] = pack8(f);
                }
                fence_async_smem();
            }
            mbar_arrive(tdone + s);
        };
        auto epilogue = [&](int it) {
            const int ab = it & 1;
            ok = ok && mbar_wait(acc_full + ab, (it >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + ab * C::ACC + (static_cast<uint32_t>(sp * 32) << 16);
            uint32_t v[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t r[16];
                tmem_ld16(acc + c0, r);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[c0 + e] = r[e];
            }
            uint32_t zr[16];
            tmem_ld16(acc + D, zr);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(acc_empty + ab);
            const int tile = blockIdx.x + it * gridDim.x;
            const int tok = tile * kTile + sp * 32 + lane;
            if (!ok || tok >= N) return;
            const float den = __uint_as_float(zr[0]);
            uint4* o = reinterpret_cast<uint4*>(out + ((size_t)bh * N + tok) * D);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 8) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float num = __uint_as_float(v[c0 + e]);
                    f[e] = normalize ? num / den : num;
                }
                o[c0 / 8] = pack8(f);
            }
        };
        if (my_tiles > 0) transform(0);
        for (int it = 0; it < my_tiles; ++it) {
            if (it + 1 < my_tiles) transform(it + 1);
            epilogue(it);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Chunked causal / prefix-mask outputs of one block
// ---------------------------------------------------------------------------
// The block's chunks are swept in order with the running state of all
// earlier keys kept in TMEM: S (fp32, M = d_k rows) and z (fp32, every column
// of a 16-column block equal to z), both seeded from the block's prefix
// record. For chunk c (C keys) and each tile of up to C queries answered
// there:
//   S_prev, z_prev -> bf16 operands (z as hi + lo rows)      [prep warps]
//   S += phi(K_c)^T V_c ;  z += phi(K_c)^T 1                   [MMA]
//   P  = phi(Q) phi(K_c)^T                                     [MMA, M = C]
//   P~ = P with keys j > lim_i zeroed, bf16; den_i = rowsum   [mask warps]
//   O  = phi(Q) S_prev + P~ V_c ; den_i += phi(Q) z_prev       [MMA]
//   out_i = O_i / den_i                                        [mask warps]
// Causal: the queries of chunk c are its own tokens, lim_i = i - cC.
// Prefix mask: the queries of bin c (floor((m_i+1)/C) = c) are gathered
// rows, lim_i = m_i - cC in [-1, C-2].
//
// Warp roles (320 threads): warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 "prep"
// (phi on the K / Q tiles, state -> operands, query gather), warps 6-9 "mask"
// (P~, epilogue). Prep runs one chunk ahead of mask; the S / z operands are
// double-buffered, the gathered query tiles too.
template <int D, int C, bool GATHER>
struct SwCfg {
    static constexpr int NB = D / 64;
    static constexpr int TILE = C * D * 2;           // one [C x D] bf16 tile
    static constexpr int NT = GATHER ? 2 : 3;        // tiles per stage: (Q,) K, V
    static constexpr int STAGES = (D == 64 && C == 64) ? 3 : 2;
    static constexpr int STAGE = NT * TILE;
    static constexpr int PT = C * C * 2;             // P~, K-major
    static constexpr int B3 = D * D * 2;             // S_prev, MN-major (x2)
    static constexpr int BZ = 16 * D * 2;            // z_hi, z_lo, 14 zero rows; K-major (x2)
    static constexpr int ONES = 16 * C * 2;          // all-ones B operand, 16 x C, K-major
    static constexpr int QG = GATHER ? 2 * TILE : 0; // gathered queries (x2)
    static constexpr int ROWS = GATHER ? 2 * 2 * C * 4 : 0;  // token / limit per row (x2)
    static constexpr int COL_S = 0, COL_Z = D, COL_P = D + 16, COL_O = D + 16 + C, COL_OZ = 2 * D + 16 + C;
    static constexpr uint32_t TMEM_COLS = (2 * D + 32 + C) <= 256 ? 256u : 512u;
    static constexpr int NBAR = 2 * STAGES + 8;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + PT + 2 * B3 + 2 * BZ + ONES + QG +
                                   ROWS + 8 * NBAR + 16;
    static constexpr int THREADS = 320;
    static constexpr int MIN_BLOCKS = (D == 64 && C == 64) ? 2 : 1;
    static_assert(C == 64 || C == 128, "chunk");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int D, int C, bool GATHER>
__global__ void __launch_bounds__(SwCfg<D, C, GATHER>::THREADS, SwCfg<D, C, GATHER>::MIN_BLOCKS)
tc_sweep_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                const __grid_constant__ CUtensorMap mV, const __nv_bfloat16* __restrict__ Qg,
                const float* __restrict__ prefix, int H, int N, int block_tokens, int nblk,
                const int32_t* __restrict__ perm, const int32_t* __restrict__ bin_start,
                const int32_t* __restrict__ mcl, int nbins, int phi, int normalize,
                __nv_bfloat16* __restrict__ out, uint32_t* __restrict__ err) {
    using CF = SwCfg<D, C, GATHER>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* pt = stages + CF::STAGES * CF::STAGE;
    uint8_t* b3 = pt + CF::PT;
    uint8_t* bz = b3 + 2 * CF::B3;
    uint8_t* ones = bz + 2 * CF::BZ;
    uint8_t* qg = ones + CF::ONES;
    int* rows = reinterpret_cast<int*>(qg + CF::QG);  // [slot][srow C | slim C]
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(rows) + CF::ROWS);
    uint64_t* empty = full + CF::STAGES;
    uint64_t* bprep = empty + CF::STAGES;
    uint64_t* bsdone = bprep + 1;
    uint64_t* bpfull = bsdone + 1;
    uint64_t* bptready = bpfull + 1;
    uint64_t* bofull = bptready + 1;
    uint64_t* bofree = bofull + 1;  // [2], one per query-tile slot
    uint64_t* bqready = bofree + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bqready + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    const int c_end = (GATHER && blk == nblk - 1) ? nbins : min(nchunks, c_begin + block_tokens / C);
    const int nci = c_end - c_begin;
    const bool relu = phi == PHI_RELU1;
    const size_t hoff = (size_t)bh * N * D;

    auto q_tiles = [&](int c) -> int {
        if (!GATHER) return c < nchunks ? 1 : 0;
        const int cnt = bin_start[(size_t)b * (nbins + 1) + c + 1] - bin_start[(size_t)b * (nbins + 1) + c];
        return (cnt + C - 1) / C;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(bprep, 128);
        mbar_init(bsdone, 1);
        mbar_init(bpfull, 1);
        mbar_init(bptready, 128);
        mbar_init(bofull, 1);
        mbar_init(bofree, 128);
        mbar_init(bofree + 1, 128);
        mbar_init(bqready, 128);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, CF::TMEM_COLS);
    if (threadIdx.x == 0) {
        if (!GATHER) tma_prefetch_map(&mQ);
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued[CF::STAGES] = {};
            for (int ci = 0; ci < nci; ++ci) {
                const int s = ci % CF::STAGES, u = ci / CF::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, CF::STAGE);
                uint8_t* st = stages + s * CF::STAGE;
                const int row = (c_begin + ci) * C;
#pragma unroll
                for (int bx = 0; bx < CF::NB; ++bx) {
                    int t = 0;
                    if (!GATHER) tma_load_3d(st + (t++) * CF::TILE + bx * C * 128, &mQ, full + s, bx * 64, row, bh);
                    tma_load_3d(st + (t++) * CF::TILE + bx * C * 128, &mK, full + s, bx * 64, row, bh);
                    tma_load_3d(st + t * CF::TILE + bx * C * 128, &mV, full + s, bx * 64, row, bh);
                }
                issued[s] = u + 1;
            }
            for (int s = 0; s < CF::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id1 = idesc_bf16(C, C, false, false);   // P = Q K^T
            constexpr uint32_t id3 = idesc_bf16(C, D, false, true);    // O = Q S
            constexpr uint32_t idz = idesc_bf16(C, 16, false, false);  // Oz = Q [z]
            constexpr uint32_t id2 = idesc_bf16(C, D, false, true);    // O += P~ V
            constexpr uint32_t id4 = idesc_bf16(D, D, true, true);     // S += K^T V
            constexpr uint32_t id5 = idesc_bf16(D, 16, true, false);   // Z += K^T 1
            const uint32_t pta = smem_u32(pt), onesa = smem_u32(ones);
            int tq = 0;
            bool ok = true;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t st = smem_u32(stages + s * CF::STAGE);
                const uint32_t kt = st + (GATHER ? 0 : CF::TILE);
                const uint32_t vt = kt + CF::TILE;
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t a = sdesc(kt + kk * 2048, C * 128, 1024);
                    mma_bf16(tmem + CF::COL_S, a, sdesc(vt + kk * 2048, C * 128, 1024), id4, 1u);
                    if (normalize)
                        mma_bf16(tmem + CF::COL_Z, a, sdesc(onesa + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024),
                                 id5, 1u);
                }
                mma_commit(bsdone);
                const uint32_t b3a = smem_u32(b3 + (ci & 1) * CF::B3);
                const uint32_t bza = smem_u32(bz + (ci & 1) * CF::BZ);
                const int ntq = q_tiles(c_begin + ci);
                for (int t = 0; t < ntq && ok; ++t, ++tq) {
                    const uint32_t qt = GATHER ? smem_u32(qg + (tq & 1) * CF::TILE) : st;
                    if (GATHER) ok = mbar_wait(bqready, tq & 1, err);
                    if (ok && tq > 0) ok = mbar_wait(bptready, (tq - 1) & 1, err);  // P read by the mask warps
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ko = (kk / 4) * (C * 128) + (kk % 4) * 32;
                        mma_bf16(tmem + CF::COL_P, sdesc(qt + ko, 16, 1024), sdesc(kt + ko, 16, 1024), id1, kk > 0);
                    }
                    mma_commit(bpfull);
                    if (tq > 0) ok = mbar_wait(bofree + ((tq - 1) & 1), ((tq - 1) >> 1) & 1, err);  // O read
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = sdesc(qt + (kk / 4) * (C * 128) + (kk % 4) * 32, 16, 1024);
                        mma_bf16(tmem + CF::COL_O, a, sdesc(b3a + kk * 2048, D * 128, 1024), id3, kk > 0);
                        if (normalize)
                            mma_bf16(tmem + CF::COL_OZ, a, sdesc(bza + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024),
                                     idz, kk > 0);
                    }
                    ok = mbar_wait(bptready, tq & 1, err);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tmem + CF::COL_O, sdesc(pta + (kk / 4) * (C * 128) + (kk % 4) * 32, 16, 1024),
                                 sdesc(vt + kk * 2048, C * 128, 1024), id2, 1u);
                    mma_commit(bofull);
                }
                mma_commit(empty + s);
            }
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        constexpr int RS = D == 128 ? 32 : 16;  // S rows per sub-partition
        const float* pre = prefix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
        {
            const uint4 one8 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
            for (int c = et; c < CF::ONES / 16; c += 128) reinterpret_cast<uint4*>(ones)[c] = one8;
            for (int c = et; c < 2 * 16 * D / 8; c += 128) {  // z operand rows 2..15 stay zero
                const int buf = c / (16 * D / 8), cc = c % (16 * D / 8);
                const int n = cc / (D / 8), col = (cc % (D / 8)) * 8;
                if (n >= 2)
                    *reinterpret_cast<uint4*>(bz + buf * CF::BZ + (col / 64) * 2048 + sw128_off(n, col % 64)) =
                        make_uint4(0, 0, 0, 0);
            }
            // seed the TMEM state with the block's prefix
            const int a = sp * RS + lane;
            const bool own = lane < RS;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t r[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 x = own ? reinterpret_cast<const float4*>(pre + (size_t)a * D + c0)[q4]
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    r[4 * q4] = __float_as_uint(x.x);
                    r[4 * q4 + 1] = __float_as_uint(x.y);
                    r[4 * q4 + 2] = __float_as_uint(x.z);
                    r[4 * q4 + 3] = __float_as_uint(x.w);
                }
                tmem_st16(tmem + CF::COL_S + lane_base + c0, r);
            }
            if (normalize) {
                uint32_t r[16];
                const uint32_t zv = own ? __float_as_uint(pre[(size_t)D * D + a]) : 0u;
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = zv;
                tmem_st16(tmem + CF::COL_Z + lane_base, r);
            }
            tmem_st_wait();
        }
        bool ok = true;
        int tq = 0;
        for (int ci = 0; ci < nci && ok; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
            uint8_t* st = stages + s * CF::STAGE;
            uint4* kt = reinterpret_cast<uint4*>(st + (GATHER ? 0 : CF::TILE));
            ok = mbar_wait(full + s, u & 1, err);
            if (!ok) break;
#pragma unroll 4
            for (int i = 0; i < CF::NB * C / 16; ++i) {
                const int p = et + 128 * i;
                const int r = (p % (C * 8)) >> 3;
                float f[8];
                unpack8(kt[p], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = r < kvalid ? phi_apply(f[e], phi) : 0.f;
                kt[p] = pack8(f);
                if (!GATHER && relu) {
                    uint4* qt = reinterpret_cast<uint4*>(st);
                    unpack8(qt[p], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = phi_relu1(f[e]);
                    qt[p] = pack8(f);
                }
            }
            if (ci > 0) {
                ok = mbar_wait(bsdone, (ci - 1) & 1, err);
                tc_fence_after();
            }
            // S_prev -> bf16 MN-major operand (rows = d_k index)
            uint8_t* b3b = b3 + (ci & 1) * CF::B3;
            if (D == 128) {
                const int a = sp * 32 + lane;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t r[64];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tmem_ld16(tmem + CF::COL_S + lane_base + 64 * h + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * j));
                    tmem_ld_wait();
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * g + e]);
                        *reinterpret_cast<uint4*>(b3b + h * (D * 128) + sw128_off(a, 8 * g)) = pack8(f);
                    }
                }
            } else {
                const int a = sp * 16 + (lane & 15);
                const int cb = lane < 16 ? 0 : 32;
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + CF::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + CF::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * g + e]);
                    *reinterpret_cast<uint4*>(b3b + sw128_off(a, cb + 8 * g)) = pack8(f);
                }
            }
            // z_prev -> rows 0 (hi) and 1 (lo) of the z operand
            if (normalize) {
                uint32_t r[16];
                tmem_ld16(tmem + CF::COL_Z + lane_base, r);
                tmem_ld_wait();
                if (lane < RS) {
                    const int a = sp * RS + lane;
                    const float zv = __uint_as_float(r[0]);
                    const __nv_bfloat16 hi = __float2bfloat16_rn(zv);
                    const __nv_bfloat16 lo = __float2bfloat16_rn(zv - __bfloat162float(hi));
                    uint8_t* base = bz + (ci & 1) * CF::BZ + (a / 64) * 2048;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(0, a % 64)) = hi;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(1, a % 64)) = lo;
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);

            if (GATHER) {
                const int ntq = q_tiles(c);
                const int qbase = bin_start[(size_t)b * (nbins + 1) + c];
                const int qend = bin_start[(size_t)b * (nbins + 1) + c + 1];
                for (int t = 0; t < ntq && ok; ++t, ++tq) {
                    const int slot = tq & 1;
                    if (tq >= 2) ok = mbar_wait(bofree + slot, ((tq >> 1) - 1) & 1, err);
                    if (!ok) break;
                    int* srow = rows + slot * 2 * C;
                    int* slim = srow + C;
                    if (et < C) {
                        const int idx = qbase + t * C + et;
                        if (idx < qend) {
                            const int i = perm[(size_t)b * N + idx];
                            srow[et] = i;
                            slim[et] = mcl[(size_t)b * N + i] - c * C;
                        } else {
                            srow[et] = -1;
                            slim[et] = -1;
                        }
                    }
                    named_bar(1, 128);
                    uint8_t* q = qg + slot * CF::TILE;
                    for (int p = et; p < C * D / 8; p += 128) {
                        const int r = p / (D / 8), col = (p % (D / 8)) * 8;
                        float f[8];
                        const int i = srow[r];
                        if (i >= 0) {
                            unpack8(ldg_stream(Qg + hoff + (size_t)i * D + col), f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = phi_apply(f[e], phi);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = 0.f;
                        }
                        *reinterpret_cast<uint4*>(q + (col / 64) * (C * 128) + sw128_off(r, col % 64)) = pack8(f);
                    }
                    fence_async_smem();
                    mbar_arrive(bqready);
                }
            }
        }
    } else {
        // ---------------- mask + epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        // M = C accumulators: C = 128 -> lane = row; C = 64 -> rows in lanes
        // 0..15, the two halves of the warp take the two column halves.
        const int i = C == 128 ? sp * 32 + lane : sp * 16 + (lane & 15);
        const int half = (C == 64 && lane >= 16) ? 1 : 0;
        bool ok = true;
        int tq = 0;
        for (int ci = 0; ci < nci && ok; ++ci) {
            const int c = c_begin + ci;
            const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
            const int ntq = q_tiles(c);
            for (int t = 0; t < ntq && ok; ++t, ++tq) {
                const int slot = tq & 1;
                ok = mbar_wait(bpfull, tq & 1, err);
                tc_fence_after();
                // the row table of a gathered tile is written before its MMAs are issued
                const int* srow = rows + slot * 2 * C;
                const int lim = GATHER ? srow[C + i] : i;
                const int tok = GATHER ? srow[i] : (i < kvalid ? c * C + i : -1);
                float rs = 0.f;
                if (C == 128) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t r[64];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tmem_ld16(tmem + CF::COL_P + lane_base + 64 * h + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * j));
                        tmem_ld_wait();
#pragma unroll
                        for (int g = 0; g < 8; ++g) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int j = 64 * h + 8 * g + e;
                                f[e] = j <= lim ? __uint_as_float(r[8 * g + e]) : 0.f;
                                rs += f[e];
                            }
                            *reinterpret_cast<uint4*>(pt + h * (C * 128) + sw128_off(i, 8 * g)) = pack8(f);
                        }
                    }
                } else {
                    uint32_t r[32];
                    tmem_ld16x2<32>(tmem + CF::COL_P + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                    tmem_ld16x2<32>(tmem + CF::COL_P + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                    tmem_ld_wait();
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 32 * half + 8 * g + e;
                            f[e] = j <= lim ? __uint_as_float(r[8 * g + e]) : 0.f;
                            rs += f[e];
                        }
                        *reinterpret_cast<uint4*>(pt + sw128_off(i, 32 * half + 8 * g)) = pack8(f);
                    }
                    rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bptready);
                // epilogue: this thread's segment of output row i
                ok = ok && mbar_wait(bofull, tq & 1, err);
                tc_fence_after();
                constexpr int SEG = C == 128 ? D : D / 2;
                uint32_t o[SEG];
#pragma unroll
                for (int j = 0; j < SEG / 16; ++j) {
                    if (C == 128)
                        tmem_ld16(tmem + CF::COL_O + lane_base + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(o + 16 * j));
                    else
                        tmem_ld16x2<D / 2>(tmem + CF::COL_O + lane_base + 16 * j,
                                           *reinterpret_cast<uint32_t(*)[16]>(o + 16 * j));
                }
                uint32_t oz[2];
                tmem_ld2(tmem + CF::COL_OZ + lane_base, oz);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(bofree + slot);
                float den = rs + __uint_as_float(oz[0]) + __uint_as_float(oz[1]);
                if (C == 64) den = __shfl_sync(0xffffffffu, den, lane & 15);
                if (ok && tok >= 0) {
                    uint4* dst = reinterpret_cast<uint4*>(out + hoff + (size_t)tok * D + half * SEG);
#pragma unroll
                    for (int g = 0; g < SEG / 8; ++g) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const float num = __uint_as_float(o[8 * g + e]);
                            f[e] = normalize ? num / den : num;
                        }
                        dst[g] = pack8(f);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CF::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [BH, N, d] bf16 viewed as 3-D; 64-column x `rows` boxes, 128-byte swizzle,
// zero fill outside the tensor.
cudaError_t make_map(CUtensorMap* map, const void* base, int d, int N, long long bh, int rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)bh};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_kv(const Problem& p, const void* k, const void* v, int tps, int nsplit, float* part,
                      uint32_t* err, cudaStream_t st) {
    CUtensorMap mk, mv;
    cudaError_t e = make_map(&mk, k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    constexpr size_t smem = KvCfg<D>::SMEM;
    e = ensure_smem<tc_kv_partial_kernel<D>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nsplit, (unsigned)p.bh());
    tc_kv_partial_kernel<D><<<grid, kTcThreads, smem, st>>>(mk, mv, p.N, tps, nsplit, p.phi, part, err);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                           uint32_t* err, cudaStream_t st) {
    CUtensorMap mq;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    constexpr size_t smem = RoCfg<D>::SMEM;
    e = ensure_smem<tc_readout_kernel<D>>(smem);
    if (e != cudaSuccess) return e;
    const int ntiles = (p.N + kTile - 1) / kTile;
    const long long want = std::max(1LL, (2LL * 148 + p.bh() - 1) / p.bh());
    const int gx = (int)std::min<long long>(ntiles, want);
    dim3 grid(gx, (unsigned)p.bh());
    tc_readout_kernel<D><<<grid, kTcThreads, smem, st>>>(mq, S, z, static_cast<__nv_bfloat16*>(out), p.N,
                                                         p.phi, p.normalize, err);
    return cudaGetLastError();
}

template <int D, int C, bool GATHER>
cudaError_t launch_chunked(const Problem& p, const void* q, const void* k, const void* v,
                           const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                           const int32_t* bins, const int32_t* mcl, int nbins, void* out, uint32_t* err,
                           cudaStream_t st) {
    if (block_tokens % C != 0) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mk, k, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), C);
    if (e != cudaSuccess) return e;
    using CF = SwCfg<D, C, GATHER>;
    constexpr size_t smem = CF::SMEM;
    e = ensure_smem<tc_sweep_kernel<D, C, GATHER>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nblk, (unsigned)p.bh());
    tc_sweep_kernel<D, C, GATHER><<<grid, CF::THREADS, smem, st>>>(
        mq, mk, mv, static_cast<const __nv_bfloat16*>(q), prefix, p.H, p.N, block_tokens, nblk, perm, bins,
        mcl, nbins, p.phi, p.normalize, static_cast<__nv_bfloat16*>(out), err);
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(const Problem& p) { return p.dtype == DT_BF16 && (p.d == 64 || p.d == 128); }

int tc_chunk(const Problem& p, int chunk) { return p.d == 128 ? 64 : chunk; }

cudaError_t tc_kv_partial(const Problem& p, const void* k, const void* v, int tps, int nsplit, float* part,
                          uint32_t* err, cudaStream_t st) {
    if (tps % kTile != 0) return cudaErrorInvalidValue;
    return p.d == 64 ? launch_kv<64>(p, k, v, tps, nsplit, part, err, st)
                     : launch_kv<128>(p, k, v, tps, nsplit, part, err, st);
}

cudaError_t tc_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                       uint32_t* err, cudaStream_t st) {
    return p.d == 64 ? launch_readout<64>(p, q, S, z, out, err, st)
                     : launch_readout<128>(p, q, S, z, out, err, st);
}

cudaError_t tc_chunked(const Problem& p, int chunk, const void* q, const void* k, const void* v,
                       const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                       const int32_t* bins, const int32_t* mcl, int nbins, void* out, uint32_t* err,
                       cudaStream_t st) {
    const int C = tc_chunk(p, chunk);
    const bool g = perm != nullptr;
#define LA_CH(D_, C_, G_) \
    return launch_chunked<D_, C_, G_>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, mcl, nbins, out, err, st)
    if (p.d == 128) {
        if (g) LA_CH(128, 64, true);
        LA_CH(128, 64, false);
    }
    if (C == 64) {
        if (g) LA_CH(64, 64, true);
        LA_CH(64, 64, false);
    }
    if (g) LA_CH(64, 128, true);
    LA_CH(64, 128, false);
#undef LA_CH
}

}  // namespace la
