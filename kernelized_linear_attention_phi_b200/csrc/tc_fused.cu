// Non-causal attention in one kernel for small problems (bf16, d = 64): one
// thread-block cluster of 8 CTAs per head.
//
// The balanced path (KV partial records, their reduction, the readout) runs
// three dependent kernels; for a few heads of a few thousand tokens each of
// them costs more in launch, prologue and pipeline fill than in data moved.
// Here the 8 CTAs of a head's cluster each take one eighth of its tokens:
//   1. KV partial: S_r = phi(K_r)^T V_r, z_r = sum phi(K_r) on the CTA's
//      tokens (the KV-summary pipeline: TMA, relu in place, MMA into TMEM,
//      fp32 column sums), kept in the CTA's shared memory;
//   2. reduction over the cluster: CTA r sums rows 8r .. 8r + 7 of S (and
//      z) over the 8 partials in rank order, reading them from the other
//      CTAs' shared memory, and writes the bf16 operand rows (and z_hi,
//      z_lo) into every CTA of the cluster; a cluster barrier before and
//      after (hardware barriers: every thread of every CTA reaches both on
//      every path);
//   3. readout of the CTA's tokens against the full S, z (the readout
//      pipeline), output tiles stored by TMA; skipped when only the KV
//      summary is asked for (readout = 0: S, z written, Q never loaded).
// The Q tiles of phase 3 are loaded while phases 1 and 2 finish (the stages
// are shared, and the first ones free up as the phase-1 MMAs complete).
//
// Warp roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 transforms, column sums, the reduction and epilogues.

#include "device.h"
#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kCluster = 8;

struct FnCfg {
    static constexpr int D = 64;
    static constexpr int TILE = kTile * D * 2;   // one [128 x 64] bf16 tile
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 2 * TILE;       // K, V (phase 1); Q (phase 3)
    static constexpr int SP = (D * D + D) * 4;   // the CTA's partial (S_r, z_r), fp32
    static constexpr int RED = 128 * 2 * 8 * 4;  // column-sum partials (phase 1, in the staging tile)
    static constexpr int BS = D * D * 2;         // S, bf16 [d_k][d_v], MN-major
    static constexpr int BZ = 16 * D * 2;        // [z_hi; z_lo; 0], K-major
    static constexpr int STG = TILE;             // output staging tile
    static constexpr int ACC = D + 16;           // readout accumulator columns per buffer
    static constexpr int COL_S = 0, COL_O = D;   // S (M = 64), then two readout buffers
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr int BARS = 3 * STAGES + 1 + 4;
    // swizzled tiles first (each 1024-byte aligned), then the fp32 scratch
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + STG + BS + BZ + SP + D * 4 + 8 * BARS + 16;
    static_assert(RED <= STG, "column-sum scratch fits the staging tile");
    // two resident CTAs per SM (a cluster then needs 4 SMs): 228 KiB per SM, 1 KiB reserved per CTA
    static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
    static_assert(STAGE % 1024 == 0 && STG % 1024 == 0 && BS % 1024 == 0 && BZ % 1024 == 0,
                  "128-byte-swizzled tiles start on 1024-byte boundaries");
    static_assert(COL_O + 2 * ACC <= (int)TMEM_COLS, "TMEM");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(D % kCluster == 0 && (D / kCluster) * (D / 8) <= 128, "row slice per CTA");
};

template <int PHI>
__global__ void __launch_bounds__(kThreads, 2)
tc_noncausal_cluster_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                            const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mOut, int N,
                            int tpc, int normalize, int readout, float* __restrict__ S_out,
                            float* __restrict__ z_out, uint32_t* __restrict__ err) {
    using C = FnCfg;
    constexpr int D = C::D;
    constexpr bool relu = PHI == PHI_RELU1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* stg = tiles + C::STAGES * C::STAGE;
    uint8_t* bS = stg + C::STG;
    uint8_t* bZ = bS + C::BS;
    float* spart = reinterpret_cast<float*>(bZ + C::BZ);  // S_r [a][v], then z_r [a]
    float* red = reinterpret_cast<float*>(stg);  // phase 1 only: the staging tile is free until phase 3
    float* csum = spart + D * D + D;
    uint64_t* full = reinterpret_cast<uint64_t*>(csum + D);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* segdone = empty + C::STAGES;
    uint64_t* acc_full = segdone + 1;   // [2]
    uint64_t* acc_empty = acc_full + 2; // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rank = blockIdx.x;  // the cluster spans blockIdx.x = 0 .. kCluster - 1
    const int bh = blockIdx.y;
    const int t0 = rank * tpc;
    const int t1 = min(N, t0 + tpc);
    const int nt = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;  // tiles of phase 1
    const int nq = readout ? nt : 0;                              // tiles of phase 3

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(tdone + s, 128);
            mbar_init(empty + s, 1);
        }
        mbar_init(segdone, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(acc_full + a, 1);
            mbar_init(acc_empty + a, 128);
        }
        fence_mbar_init();
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
        tma_prefetch_map(&mQ);
        tma_prefetch_map(&mOut);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    for (int c = threadIdx.x; c < C::BZ / 16; c += kThreads) reinterpret_cast<uint4*>(bZ)[c] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // This kernel is the first of its call: the kernel before it on the stream
    // may be the last kernel of an earlier call whose outputs are this call's
    // inputs (and that kernel lets its dependents launch early). So every warp,
    // the TMA producer included, waits for it before reading anything.
    pdl_wait();

    // Ring of stages shared by both phases: phase-1 tile i is ring index i,
    // phase-3 tile i is ring index nt + i (stage ring % STAGES, use ring / STAGES).
    if (warp == 0) {
        // ---------------- TMA producer ----------------
        int issued[C::STAGES] = {};
        bool ok = true;
        auto load = [&](int ring, int i, bool q) {
            const int s = ring % C::STAGES, u = ring / C::STAGES;
            if (u > 0 && !(ok = mbar_wait(empty + s, (u - 1) & 1, err))) return;
            uint8_t* st = tiles + s * C::STAGE;
            const int row = t0 + i * kTile;
            if (q) {
                mbar_arrive_expect_tx(full + s, C::TILE);
                tma_load_3d(st, &mQ, full + s, 0, row, bh);
            } else {
                mbar_arrive_expect_tx(full + s, 2 * C::TILE);
                tma_load_3d(st, &mK, full + s, 0, row, bh);
                tma_load_3d(st + C::TILE, &mV, full + s, 0, row, bh);
            }
            issued[s] = u + 1;
        };
        if (lane == 0) {
            for (int i = 0; i < nt && ok; ++i) load(i, i, false);
            // the first Q tiles wait only for phase-1 MMAs to free their stages
            for (int i = 0; i < min(nq, C::STAGES) && ok; ++i) load(nt + i, i, true);
        }
        cluster_sync();
        cluster_sync();
        if (lane == 0) {
            for (int i = C::STAGES; i < nq && ok; ++i) load(nt + i, i, true);
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        bool ok = true;
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(D, D, true, true);  // S_r += K^T V
            for (int i = 0; i < nt && ok; ++i) {
                const int s = i % C::STAGES, u = i / C::STAGES;
                if (!(ok = mbar_wait(tdone + s, u & 1, err))) break;
                tc_fence_after();
                const uint32_t kt = smem_u32(tiles + s * C::STAGE), vt = kt + C::TILE;
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_bf16(tmem + C::COL_S, sdesc(kt + kk * 2048, kTile * 128, 1024),
                             sdesc(vt + kk * 2048, kTile * 128, 1024), id_s, (i > 0 || kk > 0) ? 1u : 0u);
                mma_commit(empty + s);
            }
            if (nt > 0) mma_commit(segdone);
            else mbar_arrive(segdone);  // no tokens: S_r is zero (the epilogue writes zeros)
        }
        cluster_sync();
        cluster_sync();
        if (lane == 0) {
            // S, z operands were written by the cluster's CTAs (generic stores)
            fence_async_smem();
            tc_fence_after();
            constexpr uint32_t id_o = idesc_bf16(128, D, false, true);    // O = phi(Q) S
            constexpr uint32_t id_z = idesc_bf16(128, 16, false, false);  // den = phi(Q) [z]
            const uint32_t sb = smem_u32(bS), zb = smem_u32(bZ);
            for (int i = 0; i < nq && ok; ++i) {
                const int ring = nt + i, s = ring % C::STAGES, u = ring / C::STAGES;
                const int ab = i & 1, ua = i >> 1;
                if (!(ok = mbar_wait(tdone + s, u & 1, err))) break;
                if (ua > 0 && !(ok = mbar_wait(acc_empty + ab, (ua - 1) & 1, err))) break;
                tc_fence_after();
                const uint32_t qt = smem_u32(tiles + s * C::STAGE);
                const uint32_t acc = tmem + C::COL_O + ab * C::ACC;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = sdesc(qt + kk * 32, 16, 1024);
                    mma_bf16(acc, a, sdesc(sb + kk * 2048, D * 128, 1024), id_o, kk > 0 ? 1u : 0u);
                    if (normalize) mma_bf16(acc + D, a, sdesc(zb + kk * 32, 16, 1024), id_z, kk > 0 ? 1u : 0u);
                }
                mma_commit(empty + s);
                mma_commit(acc_full + ab);
            }
        }
    } else {
        // ---------------- transforms, reduction, epilogues ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        // No early exit here: after a failed wait the code runs on without
        // waiting (see cta_abort), so the named and cluster barriers match.
        bool ok = true;
        // ---- phase 1: phi on the K tiles in place, fp32 column sums (the
        // thread owns column group (et % 8) xor ((et / 8) % 8) of every tile)
        float zk[8], cv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) zk[e] = cv[e] = 0.f;
        for (int i = 0; i < nt; ++i) {
            const int s = i % C::STAGES, u = i / C::STAGES;
            ok = mbar_wait(full + s, u & 1, err) && ok;
            const int valid = min(kTile, t1 - (t0 + i * kTile));
            uint4* kt = reinterpret_cast<uint4*>(tiles + s * C::STAGE);
            const uint4* vt = reinterpret_cast<const uint4*>(tiles + s * C::STAGE + C::TILE);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int p = et + 128 * q, r = p >> 3;  // chunk, token row
                uint4 wk = kt[p];
                if (r < valid) {
                    if (relu) {
                        wk = relu_x8(wk);  // S = relu(K)^T V + 1 (x) colsum(V), z = colsum(relu K) + count
                        kt[p] = wk;
                    } else if (PHI == PHI_ELU1) {
                        wk = phi_elu1_x8(wk);
                        kt[p] = wk;
                    }
                } else {
                    wk = make_uint4(0, 0, 0, 0);
                    kt[p] = wk;
                }
                float f[8];
                unpack8(wk, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) zk[e] += f[e];
                if (relu) {  // V rows past the head's end are zero (TMA fill)
                    unpack8(vt[p], f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) cv[e] += f[e];
                }
            }
            fence_async_smem();
            mbar_arrive(tdone + s);
        }
        // the 16 threads of a column group add up their parts; in a warp,
        // lanes l, l^9, l^18, l^27 hold the same group
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            zk[e] += __shfl_xor_sync(0xffffffffu, zk[e], 9);
            zk[e] += __shfl_xor_sync(0xffffffffu, zk[e], 18);
            cv[e] += __shfl_xor_sync(0xffffffffu, cv[e], 9);
            cv[e] += __shfl_xor_sync(0xffffffffu, cv[e], 18);
        }
        const int wq = et >> 5;
        if (lane < 8) {
            const int g = lane ^ ((4 * wq) & 7);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                red[(wq * 8 + g) * 16 + e] = zk[e];
                red[(wq * 8 + g) * 16 + 8 + e] = cv[e];
            }
        }
        named_bar(1, 128);
        if (et < D) {
            const int g = et / 8, e = et % 8;
            float zs = relu ? (float)max(0, t1 - t0) : 0.f;
            float cs = 0.f;
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {  // fixed order
                zs += red[(w4 * 8 + g) * 16 + e];
                cs += red[(w4 * 8 + g) * 16 + 8 + e];
            }
            spart[D * D + et] = zs;
            csum[et] = relu ? cs : 0.f;
        }
        named_bar(1, 128);
        // S_r rows from TMEM (M = 64: rows in lanes 0..15, the warp halves
        // take the column halves), plus colsum(V) for relu+1
        ok = mbar_wait(segdone, 0, err) && ok;
        tc_fence_after();
        {
            const int a = sp * 16 + (lane & 15);
            const int c0 = 32 * (lane >> 4);
            uint32_t v[32];
            tmem_ld16x2<32>(tmem + C::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(v));
            tmem_ld16x2<32>(tmem + C::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                spart[a * D + c0 + e] = (nt > 0 ? __uint_as_float(v[e]) : 0.f) + csum[c0 + e];
        }
        tc_fence_before();
        cluster_sync();  // every CTA's partial is complete
        // ---- phase 2: rows 8 rank .. 8 rank + 7 of S (and those entries of
        // z) summed over the partials in rank order, written as operands into
        // every CTA of the cluster (and in fp32 to S_out, z_out)
        constexpr int RPC = D / kCluster;  // rows per CTA
        if (et < RPC * (D / 8)) {
            const int a = rank * RPC + et / (D / 8), c = (et % (D / 8)) * 8;
            float f[8] = {};
#pragma unroll
            for (int r2 = 0; r2 < kCluster; ++r2) {
                const uint32_t base = cluster_addr(spart + a * D + c, r2);
                const float4 x0 = ld_cluster_f4(base), x1 = ld_cluster_f4(base + 16);
                f[0] += x0.x; f[1] += x0.y; f[2] += x0.z; f[3] += x0.w;
                f[4] += x1.x; f[5] += x1.y; f[6] += x1.z; f[7] += x1.w;
            }
            if (S_out != nullptr) {
                float4* o = reinterpret_cast<float4*>(S_out + (size_t)bh * D * D + (size_t)a * D + c);
                o[0] = make_float4(f[0], f[1], f[2], f[3]);
                o[1] = make_float4(f[4], f[5], f[6], f[7]);
            }
            const uint4 w8 = pack8(f);
#pragma unroll
            for (int r2 = 0; r2 < kCluster; ++r2) st_cluster_u4(cluster_addr(bS + sw128_off(a, c), r2), w8);
        } else if (et < RPC * (D / 8) + RPC && normalize) {
            const int a = rank * RPC + (et - RPC * (D / 8));
            float zv = 0.f;
#pragma unroll
            for (int r2 = 0; r2 < kCluster; ++r2) zv += ld_cluster_f(cluster_addr(spart + D * D + a, r2));
            if (z_out != nullptr) z_out[(size_t)bh * D + a] = zv;
            const __nv_bfloat16 zh = __float2bfloat16_rn(zv);
            const __nv_bfloat16 zl = __float2bfloat16_rn(zv - __bfloat162float(zh));
            for (int r2 = 0; r2 < kCluster; ++r2) {
                st_cluster_u16(cluster_addr(bZ + sw128_off(0, a), r2), __bfloat16_as_ushort(zh));
                st_cluster_u16(cluster_addr(bZ + sw128_off(1, a), r2), __bfloat16_as_ushort(zl));
            }
        } else if (et < RPC * (D / 8) + RPC && z_out != nullptr) {
            const int a = rank * RPC + (et - RPC * (D / 8));
            float zv = 0.f;
            for (int r2 = 0; r2 < kCluster; ++r2) zv += ld_cluster_f(cluster_addr(spart + D * D + a, r2));
            z_out[(size_t)bh * D + a] = zv;
        }
        asm volatile("fence.proxy.async;" ::: "memory");  // the operands are read by MMAs
        cluster_sync();  // every CTA's operands are complete; no remote access follows
        // ---- phase 3: readout of the CTA's tokens
        auto transform = [&](int i) {
            const int ring = nt + i, s = ring % C::STAGES, u = ring / C::STAGES;
            ok = ok && mbar_wait(full + s, u & 1, err);
            if (ok && PHI != PHI_IDENTITY) {
                uint4* qt = reinterpret_cast<uint4*>(tiles + s * C::STAGE);
#pragma unroll
                for (int q = 0; q < 8; ++q) qt[et + 128 * q] = phi8<PHI>(qt[et + 128 * q]);
            }
            fence_async_smem();
            mbar_arrive(tdone + s);
        };
        auto epilogue = [&](int i) {
            const int ab = i & 1;
            ok = ok && mbar_wait(acc_full + ab, (i >> 1) & 1, err);
            tc_fence_after();
            const uint32_t acc = tmem + C::COL_O + ab * C::ACC + lane_base;
            uint32_t v[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) tmem_ld16(acc + c0, *reinterpret_cast<uint32_t(*)[16]>(v + c0));
            uint32_t zr[2];
            tmem_ld2(acc + D, zr);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(acc_empty + ab);
            if (et == 0) bulk_wait_read0();  // the previous tile's store has read the staging tile
            named_bar(2, 128);
            const int r = sp * 32 + lane;  // row of the tile
            const float inv = normalize ? __frcp_rn(__uint_as_float(zr[0]) + __uint_as_float(zr[1])) : 1.0f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 8) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[c0 + e]) * inv;
                *reinterpret_cast<uint4*>(stg + sw128_off(r, c0)) = pack8(f);
            }
            fence_async_smem();
            named_bar(2, 128);
            if (et == 0 && ok) {
                tma_store_3d(&mOut, stg, 0, t0 + i * kTile, bh);
                bulk_commit();
            }
        };
        if (nq > 0) transform(0);
        for (int i = 0; i < nq; ++i) {
            if (i + 1 < nq) transform(i + 1);
            epilogue(i);
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

template <int PHI>
cudaError_t launch_fused(const Problem& p, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mq,
                         const CUtensorMap& mo, int tpc, int readout, float* S, float* z, uint32_t* err,
                         cudaStream_t st) {
    cudaError_t e = ensure_smem<tc_noncausal_cluster_kernel<PHI>>(FnCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_cluster_pdl(tc_noncausal_cluster_kernel<PHI>, dim3(kCluster, (unsigned)p.bh()), dim3(kThreads),
                              FnCfg::SMEM, st, (unsigned)kCluster, mk, mv, mq, mo, p.N, tpc, p.normalize, readout, S,
                              z, err);
}

}  // namespace

bool tc_noncausal_fused_supported(const Problem& p) {
    // one wave of 8-CTA clusters, one per head (a B200 holds 33 at two CTAs
    // per SM; measured 36 heads, two waves, at 36.9 us here against 35.8 us
    // on the three-kernel path), at most 1024 tokens per CTA (beyond that
    // the balanced three-kernel path spreads better)
    return p.dtype == DT_BF16 && p.d == FnCfg::D && p.N <= 8 * 1024 &&
           p.bh() <= max_active_clusters(kCluster, kThreads, FnCfg::SMEM);
}

cudaError_t tc_noncausal_fused(const Problem& p, const void* q, const void* k, const void* v, void* out, float* S,
                               float* z, uint32_t* err, cudaStream_t st) {
    if (!tc_noncausal_fused_supported(p)) return cudaErrorInvalidValue;
    constexpr int D = FnCfg::D;
    // KV summary only (no out): the Q and output maps are never used and
    // are encoded over K
    const int readout = out != nullptr ? 1 : 0;
    if (!readout && (S == nullptr || z == nullptr)) return cudaErrorInvalidValue;
    CUtensorMap mk, mv, mq, mo;
    cudaError_t e = make_map(&mk, k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mq, readout ? q : k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mo, readout ? out : k, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    const int tpc = ((p.N + kCluster - 1) / kCluster + kTile - 1) / kTile * kTile;  // tokens per CTA
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1: return launch_fused<PHI_RELU1>(p, mk, mv, mq, mo, tpc, readout, S, z, err, st);
        case PHI_ELU1: return launch_fused<PHI_ELU1>(p, mk, mv, mq, mo, tpc, readout, S, z, err, st);
        default: return launch_fused<PHI_IDENTITY>(p, mk, mv, mq, mo, tpc, readout, S, z, err, st);
    }
}

}  // namespace la
