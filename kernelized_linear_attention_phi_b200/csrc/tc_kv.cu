// KV summary and readout on tcgen05 tensor cores (bf16, d = 64 or 128).
//
// KV summary ("nx_f32_linear_attention.nx source", KV-summary loop):
//   S = phi(K)^T V and z = phi(K)^T 1 over a token range, as MMAs with the
//   tokens as the contraction dimension; TMA stages 128-token K and V tiles
//   in shared memory (128-byte swizzle). For phi = relu+1 the K operand is
//   relu(K), which is exact in bf16, and the "+1" is added exactly:
//   S = relu(K)^T V + 1 (x) colsum(V) and z = relu(K)^T 1 + count, where
//   colsum(V) comes from an MMA with an all-ones A operand. Accumulation is
//   fp32 in TMEM throughout, so S and z carry no bf16 rounding of phi(K).
// Readout (nx source, per-query loop):
//   out = phi(Q) S / (phi(Q) . z): MMA with M = 128 tokens, N = d_v,
//   K = d_k against S (bf16, MN-major) plus an N = 16 MMA against
//   [z_hi; z_lo] for the denominator; TMEM accumulators double-buffered; the
//   epilogue scales each row by 1 / den and stores bf16.
//
// Both kernels use a balanced split: a 1-D grid cuts the flattened sequence
// of (head, 128-token tile) pairs into equal contiguous ranges, so every SM
// gets the same number of tiles whatever B*H and N are. A range can cross a
// head boundary; the KV summary then writes one partial record per head it
// touches (reduced per head afterwards in a fixed order), the readout
// converts the next head's S into its other operand buffer.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues MMAs, warps 2-5 transform tiles and run the epilogues.

#include <algorithm>

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {

KvBalanced kv_balanced_plan(const Problem& p) {
    KvBalanced w;
    w.tph = (p.N + tc::kTile - 1) / tc::kTile;
    w.total = p.bh() * w.tph;
    w.G = (int)std::min<long long>(w.total, 148);
    const long long per = (w.total + w.G - 1) / w.G;  // most tiles a CTA gets
    w.K = (int)std::min<long long>(p.bh(), (per + w.tph - 1) / w.tph + 1);
    return w;
}

namespace {

using namespace tc;

constexpr int kThreads = 192;

__host__ __device__ __forceinline__ long long range_lo(long long total, int G, long long c) {
    return c * total / G;
}

// The CTA of a balanced split whose range holds tile t.
__device__ __forceinline__ int cta_of(const KvBalanced& w, long long t) {
    long long c = t * w.G / w.total;
    while (c + 1 < w.G && range_lo(w.total, w.G, c + 1) <= t) ++c;
    while (c > 0 && range_lo(w.total, w.G, c) > t) --c;
    return (int)c;
}

// What one CTA of the KV-summary kernel covers: either one block of one head
// (grid = blocks x heads) or one range of the balanced split (1-D grid).
struct KvWork {
    int balanced;
    int block_tokens, nblk;  // blocks mode
    KvBalanced b;            // balanced mode
};

struct Seg {
    int bh, t0, t1;  // head and token range [t0, t1)
    int slot;        // record slot
};

__device__ __forceinline__ int kv_nseg(const KvWork& w) {
    if (!w.balanced) return 1;
    const long long lo = range_lo(w.b.total, w.b.G, blockIdx.x);
    const long long hi = range_lo(w.b.total, w.b.G, blockIdx.x + 1);
    return hi > lo ? (int)((hi - 1) / w.b.tph - lo / w.b.tph + 1) : 0;
}

__device__ __forceinline__ Seg kv_seg(const KvWork& w, int N, int j) {
    Seg s;
    if (!w.balanced) {
        s.bh = blockIdx.y;
        s.t0 = blockIdx.x * w.block_tokens;
        s.t1 = min(N, s.t0 + w.block_tokens);
        s.slot = blockIdx.y * w.nblk + blockIdx.x;
    } else {
        const long long lo = range_lo(w.b.total, w.b.G, blockIdx.x);
        const long long hi = range_lo(w.b.total, w.b.G, blockIdx.x + 1);
        const long long h = lo / w.b.tph + j;
        const long long tb = max(lo, h * w.b.tph) - h * w.b.tph;
        const long long te = min(hi, (h + 1) * w.b.tph) - h * w.b.tph;
        s.bh = (int)h;
        s.t0 = (int)(tb * kTile);
        s.t1 = (int)min((long long)N, te * kTile);
        s.slot = blockIdx.x * w.b.K + j;
    }
    return s;
}

// ---------------------------------------------------------------------------
// KV summary
// ---------------------------------------------------------------------------
template <int D>
struct KvCfg {
    static constexpr int NB = D / 64;                 // 64-column boxes per tile
    static constexpr int TILE = kTile * D * 2;        // bytes of a K or V tile
    static constexpr int STAGES = D == 64 ? 4 : 3;
    static constexpr int ONES = kTile * 128;          // all-ones operand
    static constexpr int COL_S = 0, COL_CS = D, COL_Z = 2 * D;
    static constexpr uint32_t TMEM_COLS = (2 * D + 16) <= 256 ? 256u : 512u;
    static constexpr int BARS = 3 * STAGES + 1;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * 2 * TILE + ONES + 8 * BARS + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_kv_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV, int N,
             KvWork w, int phi, float* __restrict__ part, uint32_t* __restrict__ err) {
    using C = KvCfg<D>;
    constexpr size_t REC = (size_t)D * D + D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* ones = tiles + C::STAGES * 2 * C::TILE;
    uint64_t* full = reinterpret_cast<uint64_t*>(ones + C::ONES);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* segdone = empty + C::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(segdone + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nseg = kv_nseg(w);
    const bool relu = phi == PHI_RELU1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, 1);
        }
        mbar_init(segdone, 1);
        fence_mbar_init();
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    {
        const uint4 one8 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (int c = threadIdx.x; c < C::ONES / 16; c += kThreads) reinterpret_cast<uint4*>(ones)[c] = one8;
        fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued[C::STAGES] = {};
            int it = 0;
            bool ok = true;
            for (int j = 0; j < nseg && ok; ++j) {
                const Seg sg = kv_seg(w, N, j);
                const int nt = (sg.t1 - sg.t0 + kTile - 1) / kTile;
                for (int i = 0; i < nt; ++i, ++it) {
                    const int s = it % C::STAGES, u = it / C::STAGES;
                    if (u > 0 && !(ok = mbar_wait(empty + s, (u - 1) & 1, err))) break;
                    mbar_arrive_expect_tx(full + s, 2 * C::TILE);
                    uint8_t* kt = tiles + s * 2 * C::TILE;
                    const int row = sg.t0 + i * kTile;
#pragma unroll
                    for (int b = 0; b < C::NB; ++b) {
                        tma_load_3d(kt + b * kTile * 128, &mK, full + s, b * 64, row, sg.bh);
                        tma_load_3d(kt + C::TILE + b * kTile * 128, &mV, full + s, b * 64, row, sg.bh);
                    }
                    issued[s] = u + 1;
                }
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(D, D, true, true);     // S += K^T V
            constexpr uint32_t id_cs = idesc_bf16(64, D, true, true);   // rows = colsum(V)
            constexpr uint32_t id_z = idesc_bf16(D, 16, true, false);   // z += K^T 1
            const uint32_t ob = smem_u32(ones);
            int it = 0;
            bool ok = true;
            for (int j = 0; j < nseg && ok; ++j) {
                const Seg sg = kv_seg(w, N, j);
                const int nt = (sg.t1 - sg.t0 + kTile - 1) / kTile;
                for (int i = 0; i < nt; ++i, ++it) {
                    const int s = it % C::STAGES, u = it / C::STAGES;
                    if (!(ok = mbar_wait(tdone + s, u & 1, err))) break;
                    tc_fence_after();
                    const uint32_t kt = smem_u32(tiles + s * 2 * C::TILE);
                    const uint32_t vt = kt + C::TILE;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t a = sdesc(kt + kk * 2048, kTile * 128, 1024);
                        const uint64_t b = sdesc(vt + kk * 2048, kTile * 128, 1024);
                        mma_bf16(tmem + C::COL_S, a, b, id_s, acc);
                        if (relu) mma_bf16(tmem + C::COL_CS, sdesc(ob + kk * 2048, kTile * 128, 1024), b, id_cs, acc);
                        mma_bf16(tmem + C::COL_Z, a, sdesc(ob + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_z,
                                 acc);
                    }
                    mma_commit(empty + s);
                }
                mma_commit(segdone);
            }
        }
    } else {
        const int et = threadIdx.x - 64;  // 0..127
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        int it = 0;
        bool ok = true;
        for (int j = 0; j < nseg && ok; ++j) {
            const Seg sg = kv_seg(w, N, j);
            const int nt = (sg.t1 - sg.t0 + kTile - 1) / kTile;
            for (int i = 0; i < nt; ++i, ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (!(ok = mbar_wait(full + s, u & 1, err))) break;
                const int valid = min(kTile, sg.t1 - (sg.t0 + i * kTile));
                if (relu || valid < kTile) {
                    uint4* kt = reinterpret_cast<uint4*>(tiles + s * 2 * C::TILE);
#pragma unroll
                    for (int q = 0; q < C::NB * 8; ++q) {
                        const int p = et + 128 * q;       // 16-byte chunk index
                        const int r = (p & 1023) >> 3;    // token row in the tile
                        if (r < valid) {
                            if (relu) kt[p] = relu_x8(kt[p]);
                        } else {
                            kt[p] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    fence_async_smem();
                }
                mbar_arrive(tdone + s);
            }
            if (!ok) break;
            // epilogue of segment j: TMEM -> record (S rows, then z)
            ok = mbar_wait(segdone, j & 1, err);
            tc_fence_after();
            float* rec = part + (size_t)sg.slot * REC;
            const float cnt = relu ? (float)(sg.t1 - sg.t0) : 0.0f;
            if (D == 128) {
                const int a = sp * 32 + lane;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 16) {
                    uint32_t r[16], cs[16];
                    tmem_ld16(tmem + C::COL_S + lane_base + c0, r);
                    if (relu) tmem_ld16(tmem + C::COL_CS + lane_base + c0, cs);
                    tmem_ld_wait();
                    float f[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        // lanes 0..15 of the M = 64 colsum block each hold colsum(V)
                        const float c = relu ? __uint_as_float(__shfl_sync(0xffffffffu, cs[e], lane & 15)) : 0.0f;
                        f[e] = __uint_as_float(r[e]) + c;
                    }
                    float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) o[q4] = make_float4(f[4 * q4], f[4 * q4 + 1], f[4 * q4 + 2], f[4 * q4 + 3]);
                }
                uint32_t zr[16];
                tmem_ld16(tmem + C::COL_Z + lane_base, zr);
                tmem_ld_wait();
                rec[(size_t)D * D + a] = __uint_as_float(zr[0]) + cnt;
            } else {
                // M = 64 accumulators: rows in lanes 0..15; the warp halves take column halves
                const int a = sp * 16 + (lane & 15);
                const int half = lane >> 4;
                uint32_t r[32], cs[32];
                tmem_ld16x2<32>(tmem + C::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + C::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                if (relu) {
                    tmem_ld16x2<32>(tmem + C::COL_CS + lane_base, *reinterpret_cast<uint32_t(*)[16]>(cs));
                    tmem_ld16x2<32>(tmem + C::COL_CS + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(cs + 16));
                }
                uint32_t zr[2];
                tmem_ld2(tmem + C::COL_Z + lane_base, zr);
                tmem_ld_wait();
                float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + 32 * half);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    float f[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        f[e] = __uint_as_float(r[4 * q4 + e]) + (relu ? __uint_as_float(cs[4 * q4 + e]) : 0.0f);
                    o[q4] = make_float4(f[0], f[1], f[2], f[3]);
                }
                if (lane < 16) rec[(size_t)D * D + a] = __uint_as_float(zr[0]) + cnt;
            }
            tc_fence_before();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Sums the partial records of each head in CTA order (deterministic).
__global__ void kv_reduce_balanced_kernel(const float* __restrict__ part, KvBalanced w, int D,
                                          float* __restrict__ S, float* __restrict__ z) {
    const int rec4 = (D * D + D) / 4;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const long long h = blockIdx.y;
    if (e >= rec4) return;
    const int c0 = cta_of(w, h * w.tph);
    const int c1 = cta_of(w, (h + 1) * w.tph - 1);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = c0; c <= c1; ++c) {
        const long long j = h - range_lo(w.total, w.G, c) / w.tph;
        const float4 v = reinterpret_cast<const float4*>(part + ((size_t)c * w.K + j) * (size_t)(rec4 * 4))[e];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
    }
    const float r[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int idx = 4 * e + q;
        if (idx < D * D) S[(size_t)h * D * D + idx] = r[q];
        else z[(size_t)h * D + (idx - D * D)] = r[q];
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
    static constexpr int BS = D * D * 2;               // S, MN-major bf16 (x2)
    static constexpr int BZ = 16 * D * 2;              // z_hi, z_lo, 14 zero rows, K-major (x2)
    static constexpr int ACC = D + 16;                 // accumulator columns per buffer
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256 : 512;
    static constexpr int BARS = 3 * STAGES + 4;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * TILE + 2 * BS + 2 * BZ + 8 * BARS + 16;
    static constexpr int PER_SM = D == 64 ? 2 : 1;     // CTAs an SM holds (TMEM and smem)
    static_assert(SMEM * PER_SM <= 227 * 1024, "shared memory");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tc_readout_kernel(const __grid_constant__ CUtensorMap mQ, const float* __restrict__ S,
                  const float* __restrict__ z, __nv_bfloat16* __restrict__ out, int N, long long total,
                  int tph, int phi, int normalize, uint32_t* __restrict__ err) {
    using C = RoCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* bS = tiles + C::STAGES * C::TILE;
    uint8_t* bZ = bS + 2 * C::BS;
    uint64_t* full = reinterpret_cast<uint64_t*>(bZ + 2 * C::BZ);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* acc_full = empty + C::STAGES;  // [2]
    uint64_t* acc_empty = acc_full + 2;      // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const long long lo = range_lo(total, gridDim.x, blockIdx.x);
    const long long hi = range_lo(total, gridDim.x, blockIdx.x + 1);
    const int ntile = (int)(hi - lo);
    const long long h0 = lo / tph;

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
        tma_prefetch_map(&mQ);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    for (int c = threadIdx.x; c < 2 * 16 * D / 8; c += kThreads) {  // z operand rows 2..15 stay zero
        const int buf = c / (16 * D / 8), cc = c % (16 * D / 8);
        const int n = cc / (D / 8), col = (cc % (D / 8)) * 8;
        if (n >= 2)
            *reinterpret_cast<uint4*>(bZ + buf * C::BZ + (col / 64) * 2048 + sw128_off(n, col % 64)) =
                make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int it = 0; it < ntile; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, C::TILE);
                const long long g = lo + it;
#pragma unroll
                for (int b = 0; b < C::NB; ++b)
                    tma_load_3d(tiles + s * C::TILE + b * kTile * 128, &mQ, full + s, b * 64,
                                (int)(g % tph) * kTile, (int)(g / tph));
                issued[s] = u + 1;
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(128, D, false, true);
            constexpr uint32_t id_z = idesc_bf16(128, 16, false, false);
            for (int it = 0; it < ntile; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                const int ab = it & 1, ua = it >> 1;
                const int buf = (int)(((lo + it) / tph - h0) & 1);
                if (!mbar_wait(tdone + s, u & 1, err)) break;
                if (ua > 0 && !mbar_wait(acc_empty + ab, (ua - 1) & 1, err)) break;
                tc_fence_after();
                const uint32_t qt = smem_u32(tiles + s * C::TILE);
                const uint32_t sb = smem_u32(bS + buf * C::BS), zb = smem_u32(bZ + buf * C::BZ);
                const uint32_t acc = tmem + ab * C::ACC;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = sdesc(qt + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024);
                    mma_bf16(acc, a, sdesc(sb + kk * 2048, D * 128, 1024), id_s, kk > 0 ? 1u : 0u);
                    if (normalize)
                        mma_bf16(acc + D, a, sdesc(zb + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_z,
                                 kk > 0 ? 1u : 0u);
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
            const long long g = lo + it;
            const long long h = g / tph;
            if (it == 0 || g % tph == 0) {
                // first tile of a head: its S and z into operand buffer (h - h0) & 1
                uint8_t* sb = bS + ((h - h0) & 1) * C::BS;
                uint8_t* zb = bZ + ((h - h0) & 1) * C::BZ;
                const float* Sh = S + (size_t)h * D * D;
                for (int c = et; c < D * D / 8; c += 128) {
                    const int a = c / (D / 8), col = (c % (D / 8)) * 8;
                    const float4 x0 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[0];
                    const float4 x1 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[1];
                    const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    *reinterpret_cast<uint4*>(sb + (col / 64) * (D * 128) + sw128_off(a, col % 64)) = pack8(f);
                }
                for (int c = et; c < D / 8; c += 128) {
                    const int col = c * 8;
                    float fh[8], fl[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float zv = z[(size_t)h * D + col + e];
                        fh[e] = __bfloat162float(__float2bfloat16_rn(zv));
                        fl[e] = zv - fh[e];
                    }
                    uint8_t* base = zb + (col / 64) * 2048;
                    *reinterpret_cast<uint4*>(base + sw128_off(0, col % 64)) = pack8(fh);
                    *reinterpret_cast<uint4*>(base + sw128_off(1, col % 64)) = pack8(fl);
                }
            }
            const int s = it % C::STAGES, u = it / C::STAGES;
            ok = ok && mbar_wait(full + s, u & 1, err);
            if (ok && relu) {
                uint4* qt = reinterpret_cast<uint4*>(tiles + s * C::TILE);
#pragma unroll
                for (int i = 0; i < C::NB * 8; ++i) qt[et + 128 * i] = phi_relu1_x8(qt[et + 128 * i]);
            }
            fence_async_smem();
            mbar_arrive(tdone + s);
        };
        auto epilogue = [&](int it) {
            const int ab = it & 1;
            ok = ok && mbar_wait(acc_full + ab, (it >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + ab * C::ACC + (static_cast<uint32_t>(sp * 32) << 16);
            uint32_t v[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) tmem_ld16(acc + c0, *reinterpret_cast<uint32_t(*)[16]>(v + c0));
            uint32_t zr[2];
            tmem_ld2(acc + D, zr);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(acc_empty + ab);
            const long long g = lo + it;
            const int tok = (int)(g % tph) * kTile + sp * 32 + lane;
            if (!ok || tok >= N) return;
            const float inv = normalize ? __frcp_rn(__uint_as_float(zr[0]) + __uint_as_float(zr[1])) : 1.0f;
            uint4* o = reinterpret_cast<uint4*>(out + ((size_t)(g / tph) * N + tok) * D);
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 8) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[c0 + e]) * inv;
                o[c0 / 8] = pack8(f);
            }
        };
        if (ntile > 0) transform(0);
        for (int it = 0; it < ntile; ++it) {
            if (it + 1 < ntile) transform(it + 1);
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

template <int D>
cudaError_t launch_kv(const Problem& p, const void* k, const void* v, const KvWork& w, dim3 grid, float* part,
                      uint32_t* err, cudaStream_t st) {
    CUtensorMap mk, mv;
    cudaError_t e = make_map(&mk, k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    constexpr size_t smem = KvCfg<D>::SMEM;
    e = ensure_smem<tc_kv_kernel<D>>(smem);
    if (e != cudaSuccess) return e;
    tc_kv_kernel<D><<<grid, kThreads, smem, st>>>(mk, mv, p.N, w, p.phi, part, err);
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
    const int tph = (p.N + kTile - 1) / kTile;
    const long long total = p.bh() * tph;
    const int G = (int)std::min<long long>(total, 148LL * RoCfg<D>::PER_SM);
    tc_readout_kernel<D><<<G, kThreads, smem, st>>>(mq, S, z, static_cast<__nv_bfloat16*>(out), p.N, total, tph,
                                                    p.phi, p.normalize, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t tc_kv_summary(const Problem& p, const void* k, const void* v, float* part, float* S, float* z,
                          uint32_t* err, cudaStream_t st) {
    KvWork w{};
    w.balanced = 1;
    w.b = kv_balanced_plan(p);
    const dim3 grid(w.b.G);
    cudaError_t e = p.d == 64 ? launch_kv<64>(p, k, v, w, grid, part, err, st)
                              : launch_kv<128>(p, k, v, w, grid, part, err, st);
    if (e != cudaSuccess) return e;
    const int rec4 = (p.d * p.d + p.d) / 4;
    kv_reduce_balanced_kernel<<<dim3((rec4 + 127) / 128, (unsigned)p.bh()), 128, 0, st>>>(part, w.b, p.d, S, z);
    return cudaGetLastError();
}

cudaError_t tc_kv_blocks(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                         uint32_t* err, cudaStream_t st) {
    if (block_tokens % kTile != 0) return cudaErrorInvalidValue;
    KvWork w{};
    w.balanced = 0;
    w.block_tokens = block_tokens;
    w.nblk = nblk;
    const dim3 grid(nblk, (unsigned)p.bh());
    return p.d == 64 ? launch_kv<64>(p, k, v, w, grid, part, err, st)
                     : launch_kv<128>(p, k, v, w, grid, part, err, st);
}

cudaError_t tc_readout(const Problem& p, const void* q, const float* S, const float* z, void* out, uint32_t* err,
                       cudaStream_t st) {
    return p.d == 64 ? launch_readout<64>(p, q, S, z, out, err, st)
                     : launch_readout<128>(p, q, S, z, out, err, st);
}

}  // namespace la
