// Gradients of the non-causal form on tcgen05 tensor cores (bf16, d = 64 or
// 128): the derivative of out_i = phi(q_i) S / (phi(q_i) . z) with
// S = sum_j phi(k_j) v_j^T and z = sum_j phi(k_j) over all keys.
//
// With g_i = dL/dout_i, den_i = phi(q_i).z, gn_i = g_i / den_i and
// gden_i = -(g_i . out_i) / den_i (gn_i = g_i, gden_i = 0 unnormalized):
//   dq_i = phi'(q_i) * (S gn_i + gden_i z)
//   dk_j = phi'(k_j) * (G v_j + h),   dv_j = G^T phi(k_j)
// where G = sum_i phi(q_i) gn_i^T (d_k x d_v) and h = sum_i phi(q_i) gden_i.
//
// Two kernels over 128-token tiles, each split like the readout (balanced
// contiguous ranges of (head, tile) pairs):
//   tc_bwd_q_kernel   O = phi(Q) S, den = phi(Q) [z_hi; z_lo]   (MMA)
//                     out, gn, gden per row; gn overwrites the dO tile
//                     dA = GN S^T (the S operand read K-major)  (MMA)
//                     G += phi(Q)^T GN, h += phi(Q)^T [gden_hi; gden_lo]
//                                                               (MMA, TMEM)
//                     dq = phi'(q) (dA + gden z), written over the dO tile
//                     and stored; per head segment one (G, h) record in
//                     the KV summary's record format
//   (the records are summed per head by the KV summary's reduction)
//   tc_bwd_kv_kernel  dB = V G^T, dV = phi(K) G from one bf16 copy of G
//                     (read K-major and MN-major)               (MMA)
//                     dk = phi'(k) (dB + h), dv = dV, written over the K
//                     and V tiles and stored
// phi'(x) for relu+1 comes from sign bits taken before phi is applied in
// place (phi(x) rounded to bf16 no longer tells a tiny positive x from 0);
// for elu+1 it is min(phi(x), 1) (exp(x) for x <= 0, 1 above).
//
// Warp roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 tile transforms and epilogues (thread = tile row = TMEM lane).

#include <algorithm>

#include "device.h"
#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kThreads = 192;

__host__ __device__ __forceinline__ long long range_lo(long long total, int G, long long c) {
    return c * total / G;
}

// phi in place on one stage tile of 128 rows x D columns (16-byte chunks
// et, et + 128, ...), recording relu+1's sign bits per row and logical
// column group: sgn[row * D / 8 + group].
template <int D, int PHI>
__device__ __forceinline__ void phi_tile(uint8_t* tile, uint8_t* sgn, int et) {
    if constexpr (PHI != PHI_IDENTITY) {
        uint4* t = reinterpret_cast<uint4*>(tile);
#pragma unroll
        for (int i = 0; i < D / 64 * 8; ++i) {
            const int p = et + 128 * i;
            const uint4 x = t[p];
            if constexpr (PHI == PHI_RELU1) {
                const int box = p / (kTile * 8), row = (p / 8) % kTile, lc = (p % 8) ^ (row & 7);
                sgn[row * (D / 8) + box * 8 + lc] = static_cast<uint8_t>(positive_bits(x));
            }
            t[p] = phi8<PHI>(x);
        }
    }
}

// Byte offset of the 16-byte chunk holding columns c .. c + 7 of row r in a
// tile of 64-column boxes of `rows` rows each.
__device__ __forceinline__ uint32_t chunk_off(int rows, int r, int c) {
    return (uint32_t)(c / 64) * (uint32_t)(rows * 128) + sw128_off(r, c % 64);
}

// ---------------------------------------------------------------------------
// dq, and the per-segment (G, h) records
// ---------------------------------------------------------------------------
template <int D>
struct BqCfg {
    static constexpr int NB = D / 64;
    static constexpr int TILE = kTile * D * 2;     // one [128 x D] bf16 tile
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 2 * TILE;         // Q, dO
    static constexpr int BS = D * D * 2;           // S, bf16 [d_k][d_v] (x2, by head parity)
    static constexpr int BZ = 16 * D * 2;          // [z_hi; z_lo; 0], K-major (x2)
    static constexpr int BG = 16 * kTile * 2;      // [gden_hi; gden_lo; 0] over the tile, K-major (x2)
    static constexpr int SGN = kTile * D / 8;      // relu'(q) bits (per stage)
    static constexpr int ZF = 2 * D * 4;           // z in fp32 (x2)
    static constexpr int ACC = D + 16;             // O (then dA) and den columns per buffer
    static constexpr int COL_G = 2 * ACC, COL_H = COL_G + D;
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256u : 512u;
    static constexpr int BARS = 3 * STAGES + 4 * 2 + 2;
    // d = 64: dq is staged in a tile of its own, so a stage is free for the
    // next load as soon as the MMAs have read it (for relu+1 and identity,
    // whose derivative comes from the sign bits; elu+1's reads phi(Q) back,
    // so there the stage also waits for the dq epilogue). At d = 128 there is
    // no room for it and dq is written over the dO tile.
    static constexpr bool STG_DQ = D == 64;
    static constexpr int STG = STG_DQ ? TILE : 0;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + STG + 2 * BS + 2 * BZ + 2 * BG + STAGES * SGN +
                                   ZF + 8 * BARS + 16;
    // CTAs an SM holds (TMEM, shared memory and, through the launch bounds,
    // registers): at d = 64 a second CTA hides the load of a stage behind
    // the other CTA's epilogues
    static constexpr int PER_SM = D == 64 ? 2 : 1;
    static_assert(COL_H + 16 <= (int)TMEM_COLS, "TMEM");
    static_assert(PER_SM * TMEM_COLS <= 512, "TMEM per SM");
    static_assert(PER_SM * (SMEM + 1024) <= 228 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && STG % 1024 == 0 && BS % 1024 == 0, "1024-byte aligned swizzled tiles");
};

template <int D, int PHI>
__global__ void __launch_bounds__(kThreads, BqCfg<D>::PER_SM)
tc_bwd_q_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mGo,
                const __grid_constant__ CUtensorMap mDq, const float* __restrict__ S, const float* __restrict__ z,
                KvBalanced w, int normalize, float* __restrict__ part, uint32_t* __restrict__ err) {
    using C = BqCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* stg = stages + C::STAGES * C::STAGE;  // dq staging (STG_DQ)
    uint8_t* bS = stg + C::STG;
    uint8_t* bZ = bS + 2 * C::BS;
    uint8_t* bG = bZ + 2 * C::BZ;
    uint8_t* sgn = bG + 2 * C::BG;
    float* zf = reinterpret_cast<float*>(sgn + C::STAGES * C::SGN);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(zf) + C::ZF);
    uint64_t* tdone = full + C::STAGES;    // phi(Q) and the head's S, z operands ready
    uint64_t* empty = tdone + C::STAGES;   // MMA done with the stage (and, see STG_DQ, dq done with it)
    constexpr uint32_t kEmptyArrivals = (C::STG_DQ && PHI != PHI_ELU1) ? 1u : 2u;
    uint64_t* acc_full = empty + C::STAGES;  // [2] O, den
    uint64_t* gn_ready = acc_full + 2;       // [2] GN and gden operands written (O read)
    uint64_t* da_full = gn_ready + 2;        // [2] dA (and the tile's G, h terms) done
    uint64_t* acc_empty = da_full + 2;       // [2] dA read
    uint64_t* g_full = acc_empty + 2;        // the segment's G, h complete
    uint64_t* g_free = g_full + 1;           // G, h read out
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(g_free + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const long long lo = range_lo(w.total, w.G, blockIdx.x);
    const long long hi = range_lo(w.total, w.G, blockIdx.x + 1);
    const int ntile = (int)(hi - lo);
    const long long h0 = lo / w.tph;

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, kEmptyArrivals);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full + a, 1);
            mbar_init(gn_ready + a, 128);
            mbar_init(da_full + a, 1);
            mbar_init(acc_empty + a, 128);
        }
        mbar_init(g_full, 1);
        mbar_init(g_free, 128);
        fence_mbar_init();
        tma_prefetch_map(&mQ);
        tma_prefetch_map(&mGo);
        tma_prefetch_map(&mDq);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    // rows 2..15 of the z and gden operands stay zero
    for (int c = threadIdx.x; c < 2 * C::BZ / 16; c += kThreads) reinterpret_cast<uint4*>(bZ)[c] = make_uint4(0, 0, 0, 0);
    for (int c = threadIdx.x; c < 2 * C::BG / 16; c += kThreads) reinterpret_cast<uint4*>(bG)[c] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The TMA producer loads only the caller's Q and dO; every other warp
    // waits for the previous kernel (the reduction of S, z) first.
    if (warp != 0) pdl_wait();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int it = 0; it < ntile; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, C::STAGE);
                const long long g = lo + it;
                const int row = (int)(g % w.tph) * kTile, hh = (int)(g / w.tph);
                uint8_t* st = stages + s * C::STAGE;
#pragma unroll
                for (int b = 0; b < C::NB; ++b) {
                    tma_load_3d(st + b * kTile * 128, &mQ, full + s, b * 64, row, hh);
                    tma_load_3d(st + C::TILE + b * kTile * 128, &mGo, full + s, b * 64, row, hh);
                }
                issued[s] = u + 1;
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id_o = idesc_bf16(128, D, false, true);    // O = phi(Q) S
            constexpr uint32_t id_z = idesc_bf16(128, 16, false, false);  // den = phi(Q) [z]
            constexpr uint32_t id_a = idesc_bf16(128, D, false, false);   // dA = GN S^T
            constexpr uint32_t id_g = idesc_bf16(D, D, true, true);       // G += phi(Q)^T GN
            constexpr uint32_t id_h = idesc_bf16(D, 16, true, false);     // h += phi(Q)^T [gden]
            bool ok = true;
            int seg = 0;
            bool first = true;  // first tile of the current head segment
            for (int it = 0; it < ntile && ok; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                const int ab = it & 1, ua = it >> 1;
                const long long g = lo + it;
                const int buf = (int)((g / w.tph - h0) & 1);
                const bool last = it + 1 == ntile || (g + 1) % w.tph == 0;
                ok = mbar_wait(tdone + s, u & 1, err);
                if (ok && ua > 0) ok = mbar_wait(acc_empty + ab, (ua - 1) & 1, err);
                if (!ok) break;
                tc_fence_after();
                const uint32_t qt = smem_u32(stages + s * C::STAGE), gt = qt + C::TILE;
                const uint32_t sb = smem_u32(bS + buf * C::BS), zb = smem_u32(bZ + buf * C::BZ);
                const uint32_t gd = smem_u32(bG + ab * C::BG);
                const uint32_t acc = tmem + ab * C::ACC;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = sdesc(qt + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024);
                    mma_bf16(acc, a, sdesc(sb + kk * 2048, D * 128, 1024), id_o, kk > 0 ? 1u : 0u);
                    if (normalize)
                        mma_bf16(acc + D, a, sdesc(zb + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_z,
                                 kk > 0 ? 1u : 0u);
                }
                mma_commit(acc_full + ab);
                ok = mbar_wait(gn_ready + ab, ua & 1, err);
                if (!ok) break;
                tc_fence_after();
                // dA = GN S^T over the O columns (the epilogue has read O)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(acc, sdesc(gt + (kk / 4) * (kTile * 128) + (kk % 4) * 32, 16, 1024),
                             sdesc(sb + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024), id_a, kk > 0 ? 1u : 0u);
                if (first && seg > 0) {
                    ok = mbar_wait(g_free, (seg - 1) & 1, err);  // the last segment's G, h read out
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint64_t a = sdesc(qt + kk * 2048, kTile * 128, 1024);  // phi(Q)^T, MN-major
                    const uint32_t accum = (first && kk == 0) ? 0u : 1u;
                    mma_bf16(tmem + C::COL_G, a, sdesc(gt + kk * 2048, kTile * 128, 1024), id_g, accum);
                    if (normalize)
                        mma_bf16(tmem + C::COL_H, a, sdesc(gd + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_h,
                                 accum);
                }
                mma_commit(da_full + ab);
                mma_commit(empty + s);
                if (last) {
                    mma_commit(g_full);
                    ++seg;
                }
                first = last;
            }
        }
    } else {
        // ---------------- transforms and epilogues ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int r = sp * 32 + lane;  // tile row (token) of this thread in the epilogues
        bool ok = true;
        auto transform = [&](int it) {
            const long long g = lo + it;
            const long long h = g / w.tph;
            const int buf = (int)((h - h0) & 1);
            if (it == 0 || g % w.tph == 0) {
                // first tile of a head: its S and z into operand buffer buf
                uint8_t* sb = bS + buf * C::BS;
                uint8_t* zb = bZ + buf * C::BZ;
                const float* Sh = S + (size_t)h * D * D;
                for (int c = et; c < D * D / 8; c += 128) {
                    const int a = c / (D / 8), col = (c % (D / 8)) * 8;
                    const float4 x0 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[0];
                    const float4 x1 = reinterpret_cast<const float4*>(Sh + (size_t)a * D + col)[1];
                    const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    *reinterpret_cast<uint4*>(sb + chunk_off(D, a, col)) = pack8(f);
                }
                for (int c = et; c < D; c += 128) {
                    const float zv = normalize ? z[(size_t)h * D + c] : 0.f;
                    zf[buf * D + c] = zv;
                    const __nv_bfloat16 zh = __float2bfloat16_rn(zv);
                    const __nv_bfloat16 zl = __float2bfloat16_rn(zv - __bfloat162float(zh));
                    uint8_t* base = zb + (c / 64) * 2048;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(0, c % 64)) = zh;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(1, c % 64)) = zl;
                }
            }
            const int s = it % C::STAGES, u = it / C::STAGES;
            ok = ok && mbar_wait(full + s, u & 1, err);
            if (ok) phi_tile<D, PHI>(stages + s * C::STAGE, sgn + s * C::SGN, et);
            fence_async_smem();
            mbar_arrive(tdone + s);
        };
        // out, gn and gden of row r; gn overwrites g in the dO tile
        auto epi_gn = [&](int it) -> float {
            const int ab = it & 1, s = it % C::STAGES;
            ok = ok && mbar_wait(acc_full + ab, (it >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + ab * C::ACC + lane_base;
            uint32_t zr[2] = {0u, 0u};
            if (normalize) {
                tmem_ld2(acc + D, zr);
                tmem_ld_wait();
            }
            const float inv = normalize ? __frcp_rn(__uint_as_float(zr[0]) + __uint_as_float(zr[1])) : 1.0f;
            uint8_t* gt = stages + s * C::STAGE + C::TILE;
            float dot = 0.f;  // g . O (g . out = dot / den)
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t o[16];
                tmem_ld16(acc + c0, o);
                tmem_ld_wait();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint4* p = reinterpret_cast<uint4*>(gt + chunk_off(kTile, r, c0 + 8 * h2));
                    float f[8];
                    unpack8(*p, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        dot += f[e] * __uint_as_float(o[8 * h2 + e]);
                        f[e] *= inv;
                    }
                    *p = pack8(f);
                }
            }
            const float gden = normalize ? -dot * inv * inv : 0.f;
            if (normalize) {
                const __nv_bfloat16 gh = __float2bfloat16_rn(gden);
                const __nv_bfloat16 gl = __float2bfloat16_rn(gden - __bfloat162float(gh));
                uint8_t* gb = bG + ab * C::BG + (r / 64) * 2048;
                *reinterpret_cast<__nv_bfloat16*>(gb + sw128_off(0, r % 64)) = gh;
                *reinterpret_cast<__nv_bfloat16*>(gb + sw128_off(1, r % 64)) = gl;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(gn_ready + ab);
            return gden;
        };
        // dq of row r into the staging tile (STG_DQ) or over the dO tile,
        // then the tile's TMA store
        auto epi_dq = [&](int it, float gden) {
            const int ab = it & 1, s = it % C::STAGES;
            const long long g = lo + it;
            const int buf = (int)((g / w.tph - h0) & 1);
            if (C::STG_DQ) {  // the previous tile's store has read the staging tile
                if (et == 0) bulk_wait_read0();
                named_bar(2, 128);
            }
            ok = ok && mbar_wait(da_full + ab, (it >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + ab * C::ACC + lane_base;
            uint8_t* qt = stages + s * C::STAGE;
            uint8_t* gt = C::STG_DQ ? stg : qt + C::TILE;
            const uint8_t* sg = sgn + s * C::SGN + r * (D / 8);
            const float* zb = zf + buf * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t a[16];
                tmem_ld16(acc + c0, a);
                tmem_ld_wait();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int c = c0 + 8 * h2;
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(a[8 * h2 + e]) + gden * zb[c + e];
                    const uint4 pq = PHI == PHI_ELU1 ? *reinterpret_cast<const uint4*>(qt + chunk_off(kTile, r, c))
                                                     : make_uint4(0, 0, 0, 0);
                    times_phi_grad<PHI>(f, PHI == PHI_RELU1 ? sg[c / 8] : 0u, pq);
                    *reinterpret_cast<uint4*>(gt + chunk_off(kTile, r, c)) = pack8(f);
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty + ab);
            fence_async_smem();
            named_bar(2, 128);  // the dq tile is complete and no thread reads the stage any more
            if (et == 0) {
                if (ok) {
#pragma unroll
                    for (int b = 0; b < C::NB; ++b)
                        tma_store_3d(&mDq, gt + b * kTile * 128, b * 64, (int)(g % w.tph) * kTile, (int)(g / w.tph));
                    bulk_commit();
                    if (!C::STG_DQ) bulk_wait_read0();  // the store reads the stage
                }
                if (kEmptyArrivals == 2) mbar_arrive(empty + s);
            }
        };
        // the segment's (G, h) from TMEM into its record (S, z layout: G[d_k][d_v], h[d_k])
        auto epi_g = [&](int seg) {
            ok = ok && mbar_wait(g_full, seg & 1, err);
            tc_fence_after();
            float* rec = part + (size_t)(blockIdx.x * w.K + seg) * (D * D + D);
            uint32_t hr[2] = {0u, 0u};
            if (normalize) tmem_ld2(tmem + C::COL_H + lane_base, hr);
            if (D == 128) {
                const int a = sp * 32 + lane;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem + C::COL_G + lane_base + c0, v);
                    tmem_ld_wait();
                    float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        o[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                            __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
                }
                rec[(size_t)D * D + a] = __uint_as_float(hr[0]) + __uint_as_float(hr[1]);
            } else {
                // M = 64 accumulator: rows in lanes 0..15; the warp halves take column halves
                const int a = sp * 16 + (lane & 15);
                const int c0 = 32 * (lane >> 4);
                uint32_t v[32];
                tmem_ld16x2<32>(tmem + C::COL_G + lane_base, *reinterpret_cast<uint32_t(*)[16]>(v));
                tmem_ld16x2<32>(tmem + C::COL_G + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
                tmem_ld_wait();
                float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    o[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                        __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
                if (lane < 16) rec[(size_t)D * D + a] = __uint_as_float(hr[0]) + __uint_as_float(hr[1]);
            }
            tc_fence_before();
            mbar_arrive(g_free);
        };
        // gn of tile it before phi of tile it + 1: the load of it + 1 (issued
        // once tile it - 1 was stored) lands meanwhile, and the dA MMA of
        // tile it runs under the transform
        int seg = 0;
        if (ntile > 0) transform(0);
        for (int it = 0; it < ntile; ++it) {
            const float gden = epi_gn(it);
            if (it + 1 < ntile) transform(it + 1);
            epi_dq(it, gden);
            const long long g = lo + it;
            if (it + 1 == ntile || (g + 1) % w.tph == 0) epi_g(seg++);
        }
        if (et == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// dk, dv
// ---------------------------------------------------------------------------
template <int D>
struct BkCfg {
    static constexpr int NB = D / 64;
    static constexpr int TILE = kTile * D * 2;  // one [128 x D] bf16 tile
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 2 * TILE;      // K, V (then dk, dv)
    static constexpr int BGM = D * D * 2;       // G, bf16 [d_k][d_v] (x2, by head parity)
    static constexpr int HF = 2 * D * 4;        // h in fp32 (x2)
    static constexpr int SGN = kTile * D / 8;   // relu'(k) bits (per stage)
    static constexpr int ACC = 2 * D;           // dB, dV columns per buffer
    static constexpr uint32_t TMEM_COLS = D == 64 ? 256u : 512u;
    static constexpr int BARS = 3 * STAGES + 4;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * BGM + HF + STAGES * SGN + 8 * BARS + 16;
    static constexpr int PER_SM = D == 64 ? 2 : 1;  // CTAs an SM holds (TMEM and smem)
    static_assert(2 * ACC <= (int)TMEM_COLS, "TMEM");
    static_assert(SMEM * PER_SM <= 227 * 1024, "shared memory");
};

template <int D, int PHI>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_kv_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                 const __grid_constant__ CUtensorMap mDk, const __grid_constant__ CUtensorMap mDv,
                 const float* __restrict__ G, const float* __restrict__ hv, long long total, int tph,
                 uint32_t* __restrict__ err) {
    using C = BkCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* bGm = stages + C::STAGES * C::STAGE;
    float* hf = reinterpret_cast<float*>(bGm + 2 * C::BGM);
    uint8_t* sgn = reinterpret_cast<uint8_t*>(hf) + C::HF;
    uint64_t* full = reinterpret_cast<uint64_t*>(sgn + C::STAGES * C::SGN);
    uint64_t* tdone = full + C::STAGES;      // phi(K) and the head's G operand ready
    uint64_t* empty = tdone + C::STAGES;     // MMA done with the stage and dk, dv stored from it
    uint64_t* acc_full = empty + C::STAGES;  // [2]
    uint64_t* acc_empty = acc_full + 2;      // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const long long lo = range_lo(total, gridDim.x, blockIdx.x);
    const long long hi = range_lo(total, gridDim.x, blockIdx.x + 1);
    const int ntile = (int)(hi - lo);
    const long long h0 = lo / tph;

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, 2);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full + a, 1);
            mbar_init(acc_empty + a, 128);
        }
        fence_mbar_init();
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
        tma_prefetch_map(&mDk);
        tma_prefetch_map(&mDv);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp != 0) pdl_wait();  // G, h come from the previous kernel; K, V are the caller's

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued[C::STAGES] = {};
            for (int it = 0; it < ntile; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, C::STAGE);
                const long long g = lo + it;
                const int row = (int)(g % tph) * kTile, hh = (int)(g / tph);
                uint8_t* st = stages + s * C::STAGE;
#pragma unroll
                for (int b = 0; b < C::NB; ++b) {
                    tma_load_3d(st + b * kTile * 128, &mK, full + s, b * 64, row, hh);
                    tma_load_3d(st + C::TILE + b * kTile * 128, &mV, full + s, b * 64, row, hh);
                }
                issued[s] = u + 1;
            }
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id_b = idesc_bf16(128, D, false, false);  // dB = V G^T
            constexpr uint32_t id_v = idesc_bf16(128, D, false, true);   // dV = phi(K) G
            for (int it = 0; it < ntile; ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                const int ab = it & 1, ua = it >> 1;
                const int buf = (int)(((lo + it) / tph - h0) & 1);
                if (!mbar_wait(tdone + s, u & 1, err)) break;
                if (ua > 0 && !mbar_wait(acc_empty + ab, (ua - 1) & 1, err)) break;
                tc_fence_after();
                const uint32_t kt = smem_u32(stages + s * C::STAGE), vt = kt + C::TILE;
                const uint32_t gb = smem_u32(bGm + buf * C::BGM);
                const uint32_t acc = tmem + ab * C::ACC;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ko = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
                    mma_bf16(acc, sdesc(vt + ko, 16, 1024), sdesc(gb + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024),
                             id_b, kk > 0 ? 1u : 0u);
                    mma_bf16(acc + D, sdesc(kt + ko, 16, 1024), sdesc(gb + kk * 2048, D * 128, 1024), id_v,
                             kk > 0 ? 1u : 0u);
                }
                mma_commit(empty + s);
                mma_commit(acc_full + ab);
            }
        }
    } else {
        // ---------------- transforms and epilogues ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int r = sp * 32 + lane;
        bool ok = true;
        auto transform = [&](int it) {
            const long long g = lo + it;
            const long long h = g / tph;
            const int buf = (int)((h - h0) & 1);
            if (it == 0 || g % tph == 0) {
                uint8_t* gb = bGm + buf * C::BGM;
                const float* Gh = G + (size_t)h * D * D;
                for (int c = et; c < D * D / 8; c += 128) {
                    const int a = c / (D / 8), col = (c % (D / 8)) * 8;
                    const float4 x0 = reinterpret_cast<const float4*>(Gh + (size_t)a * D + col)[0];
                    const float4 x1 = reinterpret_cast<const float4*>(Gh + (size_t)a * D + col)[1];
                    const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    *reinterpret_cast<uint4*>(gb + chunk_off(D, a, col)) = pack8(f);
                }
                for (int c = et; c < D; c += 128) hf[buf * D + c] = hv[(size_t)h * D + c];
            }
            const int s = it % C::STAGES, u = it / C::STAGES;
            ok = ok && mbar_wait(full + s, u & 1, err);
            if (ok) phi_tile<D, PHI>(stages + s * C::STAGE, sgn + s * C::SGN, et);
            fence_async_smem();
            mbar_arrive(tdone + s);
        };
        auto epilogue = [&](int it) {
            const int ab = it & 1, s = it % C::STAGES;
            const long long g = lo + it;
            const int buf = (int)((g / tph - h0) & 1);
            ok = ok && mbar_wait(acc_full + ab, (it >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + ab * C::ACC + lane_base;
            uint8_t* kt = stages + s * C::STAGE;
            uint8_t* vt = kt + C::TILE;
            const uint8_t* sg = sgn + s * C::SGN + r * (D / 8);
            const float* hb = hf + buf * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t b[16], v[16];
                tmem_ld16(acc + c0, b);
                tmem_ld16(acc + D + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int c = c0 + 8 * h2;
                    float fk[8], fv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        fk[e] = __uint_as_float(b[8 * h2 + e]) + hb[c + e];
                        fv[e] = __uint_as_float(v[8 * h2 + e]);
                    }
                    uint4* pk = reinterpret_cast<uint4*>(kt + chunk_off(kTile, r, c));
                    times_phi_grad<PHI>(fk, PHI == PHI_RELU1 ? sg[c / 8] : 0u, *pk);
                    *pk = pack8(fk);
                    *reinterpret_cast<uint4*>(vt + chunk_off(kTile, r, c)) = pack8(fv);
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty + ab);
            fence_async_smem();
            named_bar(2, 128);  // dk and dv tiles complete
            if (et == 0) {
                if (ok) {
                    const int row = (int)(g % tph) * kTile, hh = (int)(g / tph);
#pragma unroll
                    for (int bx = 0; bx < C::NB; ++bx) {
                        tma_store_3d(&mDk, kt + bx * kTile * 128, bx * 64, row, hh);
                        tma_store_3d(&mDv, vt + bx * kTile * 128, bx * 64, row, hh);
                    }
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(empty + s);
            }
        };
        // the epilogue of tile it before phi of tile it + 1, whose load
        // (issued once tile it - 1 was stored) lands meanwhile
        if (ntile > 0) transform(0);
        for (int it = 0; it < ntile; ++it) {
            epilogue(it);
            if (it + 1 < ntile) transform(it + 1);
        }
        if (et == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, int PHI>
cudaError_t launch_bwd(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                       const float* S, const float* z, float* part, float* G, float* h, void* dq, void* dk,
                       void* dv, uint32_t* err, cudaStream_t st) {
    CUtensorMap mq, mg, mdq, mk, mv, mdk, mdv;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mg, dout, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mdq, dq, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mk, k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mdk, dk, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mdv, dv, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    const KvBalanced w = kv_balanced_plan(p, BqCfg<D>::PER_SM);
    e = ensure_smem<tc_bwd_q_kernel<D, PHI>>(BqCfg<D>::SMEM);
    if (e == cudaSuccess)
        e = launch_pdl(tc_bwd_q_kernel<D, PHI>, dim3(w.G), dim3(kThreads), BqCfg<D>::SMEM, st, mq, mg, mdq, S, z, w,
                       p.normalize, part, err);
    if (e == cudaSuccess) e = tc_reduce_records(p, w, part, G, h, st);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_bwd_kv_kernel<D, PHI>>(BkCfg<D>::SMEM);
    if (e != cudaSuccess) return e;
    const int Gk = plan::balanced_ctas(w.total, device_sms(), BkCfg<D>::PER_SM);
    return launch_pdl(tc_bwd_kv_kernel<D, PHI>, dim3(Gk), dim3(kThreads), BkCfg<D>::SMEM, st, mk, mv, mdk, mdv, G, h,
                      w.total, w.tph, err);
}

template <int D>
cudaError_t bwd_phi(const Problem& p, const void* q, const void* k, const void* v, const void* dout, const float* S,
                    const float* z, float* part, float* G, float* h, void* dq, void* dk, void* dv, uint32_t* err,
                    cudaStream_t st) {
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1: return launch_bwd<D, PHI_RELU1>(p, q, k, v, dout, S, z, part, G, h, dq, dk, dv, err, st);
        case PHI_ELU1: return launch_bwd<D, PHI_ELU1>(p, q, k, v, dout, S, z, part, G, h, dq, dk, dv, err, st);
        default: return launch_bwd<D, PHI_IDENTITY>(p, q, k, v, dout, S, z, part, G, h, dq, dk, dv, err, st);
    }
}

}  // namespace

size_t tc_backward_record_slots(const Problem& p) {
    const KvBalanced w = kv_balanced_plan(p, p.d == 64 ? BqCfg<64>::PER_SM : BqCfg<128>::PER_SM);
    return (size_t)w.G * w.K;
}

cudaError_t tc_noncausal_backward(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                  const float* S, const float* z, float* part, float* G, float* h, void* dq,
                                  void* dk, void* dv, uint32_t* err, cudaStream_t st) {
    return p.d == 64 ? bwd_phi<64>(p, q, k, v, dout, S, z, part, G, h, dq, dk, dv, err, st)
                     : bwd_phi<128>(p, q, k, v, dout, S, z, part, G, h, dq, dk, dv, err, st);
}

}  // namespace la
