// KV summary and readout on tcgen05 tensor cores (bf16, d = 64 or 128).
//
// KV summary ("nx_f32_linear_attention.nx source", KV-summary loop):
//   S = phi(K)^T V over a token range as MMAs with the tokens as the
//   contraction dimension; TMA stages 128-token K and V tiles in shared
//   memory (128-byte swizzle). For phi = relu+1 the K operand is relu(K),
//   which is exact in bf16, and the "+1" is added exactly:
//   S = relu(K)^T V + 1 (x) colsum(V) and z = sum relu(K) + count. The
//   column sums of relu(K) and V are fp32 sums taken by the warps that
//   prepare each tile; S accumulates in fp32 in TMEM. So S and z carry no
//   bf16 rounding of phi(K). For phi = elu+1 (no such split) the K operand
//   is phi(K) rounded to bf16 and z sums those values.
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

#include "device.h"
#include "launch_util.h"
#include "plan.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {

static_assert(plan::kTileTokens == tc::kTile, "the plans and the kernels tile tokens alike");

KvBalanced kv_balanced_plan(const Problem& p, int per_sm) { return plan::kv_balanced_plan(p, device_sms(), per_sm); }

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
    int bpc;                 // blocks mode: consecutive blocks per CTA (1 or 2)
    KvBalanced b;            // balanced mode
};

struct Seg {
    int bh, t0, t1;  // head and token range [t0, t1)
    int slot;        // record slot
};

__device__ __forceinline__ int kv_nseg(const KvWork& w) {
    if (!w.balanced) return max(0, min(w.bpc, w.nblk - (int)blockIdx.x * w.bpc));
    const long long lo = range_lo(w.b.total, w.b.G, blockIdx.x);
    const long long hi = range_lo(w.b.total, w.b.G, blockIdx.x + 1);
    return hi > lo ? (int)((hi - 1) / w.b.tph - lo / w.b.tph + 1) : 0;
}

__device__ __forceinline__ Seg kv_seg(const KvWork& w, int N, int j) {
    Seg s;
    if (!w.balanced) {
        const int blk = blockIdx.x * w.bpc + j;
        s.bh = blockIdx.y;
        s.t0 = blk * w.block_tokens;
        s.t1 = min(N, s.t0 + w.block_tokens);
        s.slot = blockIdx.y * w.nblk + blk;
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
template <int D, bool SCAN = false>
struct KvCfg {
    static constexpr int NB = D / 64;                 // 64-column boxes per tile
    static constexpr int TILE = kTile * D * 2;        // bytes of a K or V tile
    // with the in-cluster scan (short blocks, several CTAs per SM) two stages
    static constexpr int STAGES = SCAN ? 3 : (D == 64 ? 4 : 3);
    static constexpr int RED = 128 * 2 * NB * 8 * 4 + D * 4;  // per-thread column sums, colsum(V)
    static constexpr uint32_t TMEM_COLS = D <= 64 ? 64u : 128u;
    static constexpr int BARS = 3 * STAGES + 1;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * 2 * TILE + RED + 8 * BARS + 16;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    // two resident CTAs per SM with the in-cluster scan: 228 KiB per SM, 1 KiB reserved per CTA
    static_assert(!SCAN || 2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
};

// SCAN (blocks mode, one cluster of the CTAs of a head, each taking bpc
// consecutive blocks): the block records are replaced by their exclusive
// prefix over the head's blocks, computed across the cluster after its
// barrier (see the end of the kernel); S_total, z_total (nullable) receive
// the head's total.
template <int D, int PHI, bool SCAN = false>
__global__ void __launch_bounds__(kThreads, SCAN ? 2 : 1)
tc_kv_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV, int N,
             KvWork w, float* __restrict__ part, uint32_t* __restrict__ err, float* __restrict__ S_total,
             float* __restrict__ z_total) {
    using C = KvCfg<D, SCAN>;
    constexpr size_t REC = (size_t)D * D + D;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    float* red = reinterpret_cast<float*>(tiles + C::STAGES * 2 * C::TILE);
    float* csum = red + 128 * 2 * C::NB * 8;
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + C::RED);
    uint64_t* tdone = full + C::STAGES;
    uint64_t* empty = tdone + C::STAGES;
    uint64_t* segdone = empty + C::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(segdone + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nseg = kv_nseg(w);
    constexpr bool relu = PHI == PHI_RELU1;
    constexpr bool elu = PHI == PHI_ELU1;

    if (threadIdx.x == 0) {
        cta_abort_reset();
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();

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
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(D, D, true, true);  // S += K^T V
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
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_bf16(tmem, sdesc(kt + kk * 2048, kTile * 128, 1024),
                                 sdesc(vt + kk * 2048, kTile * 128, 1024), id_s, (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(empty + s);
                }
                mma_commit(segdone);
            }
        }
    } else {
        const int et = threadIdx.x - 64;  // 0..127
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        // The thread always touches the same 16-byte chunk position of each
        // 128-byte row, so within a 64-column box it owns one group of 8
        // columns, (et % 8) xor ((et / 8) % 8); the column sums below rely
        // on that.
        // No early exit here: after a failed wait the loop runs on without
        // waiting (see cta_abort), so the named barriers stay matched.
        int it = 0;
        for (int j = 0; j < nseg; ++j) {
            const Seg sg = kv_seg(w, N, j);
            const int nt = (sg.t1 - sg.t0 + kTile - 1) / kTile;
            float zk[C::NB][8], cv[C::NB][8];  // column sums of the K operand and of V
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
#pragma unroll
                for (int e = 0; e < 8; ++e) zk[b][e] = cv[b][e] = 0.f;
            for (int i = 0; i < nt; ++i, ++it) {
                const int s = it % C::STAGES, u = it / C::STAGES;
                mbar_wait(full + s, u & 1, err);
                const int valid = min(kTile, sg.t1 - (sg.t0 + i * kTile));
                uint4* kt = reinterpret_cast<uint4*>(tiles + s * 2 * C::TILE);
                const uint4* vt = reinterpret_cast<const uint4*>(tiles + s * 2 * C::TILE + C::TILE);
#pragma unroll
                for (int q = 0; q < C::NB * 8; ++q) {
                    const int p = et + 128 * q;      // 16-byte chunk index
                    const int b = q / 8;             // 64-column box
                    const int r = (p & 1023) >> 3;   // token row in the tile
                    uint4 wk = kt[p];
                    if (r < valid) {
                        if (relu) {
                            wk = relu_x8(wk);
                            kt[p] = wk;
                        } else if (elu) {  // no exact split: phi(K) itself, rounded to bf16
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
                    for (int e = 0; e < 8; ++e) zk[b][e] += f[e];
                    if (relu) {  // rows past the end of the head are zero in V (TMA fill)
                        unpack8(vt[p], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) cv[b][e] += f[e];
                    }
                }
                fence_async_smem();
                mbar_arrive(tdone + s);
            }
            // column sums: the 16 threads of a column group add up their parts;
            // in a warp, lanes l, l^9, l^18, l^27 hold the same group
#pragma unroll
            for (int b = 0; b < C::NB; ++b)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    zk[b][e] += __shfl_xor_sync(0xffffffffu, zk[b][e], 9);
                    zk[b][e] += __shfl_xor_sync(0xffffffffu, zk[b][e], 18);
                    cv[b][e] += __shfl_xor_sync(0xffffffffu, cv[b][e], 9);
                    cv[b][e] += __shfl_xor_sync(0xffffffffu, cv[b][e], 18);
                }
            const int wq = et >> 5;  // warp of the group (0..3)
            if (lane < 8) {
                const int g = lane ^ ((4 * wq) & 7);  // group of lanes 0..7 in this warp
#pragma unroll
                for (int b = 0; b < C::NB; ++b)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        red[((wq * C::NB + b) * 8 + g) * 16 + e] = zk[b][e];
                        red[((wq * C::NB + b) * 8 + g) * 16 + 8 + e] = cv[b][e];
                    }
            }
            named_bar(1, 128);
            float* rec = part + (size_t)sg.slot * REC;
            if (et < D) {
                const int b = et / 64, g = (et % 64) / 8, e = et % 8;
                float zs = relu ? (float)(sg.t1 - sg.t0) : 0.f;
                float cs = 0.f;
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) {  // fixed order
                    zs += red[((w4 * C::NB + b) * 8 + g) * 16 + e];
                    cs += red[((w4 * C::NB + b) * 8 + g) * 16 + 8 + e];
                }
                rec[(size_t)D * D + et] = zs;
                csum[et] = relu ? cs : 0.f;
            }
            named_bar(1, 128);
            // epilogue of segment j: S rows from TMEM (+ colsum(V) for phi = relu+1)
            mbar_wait(segdone, j & 1, err);
            tc_fence_after();
            if (D == 128) {
                const int a = sp * 32 + lane;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld16(tmem + lane_base + c0, r);
                    tmem_ld_wait();
                    float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        o[q4] = make_float4(__uint_as_float(r[4 * q4]) + csum[c0 + 4 * q4],
                                            __uint_as_float(r[4 * q4 + 1]) + csum[c0 + 4 * q4 + 1],
                                            __uint_as_float(r[4 * q4 + 2]) + csum[c0 + 4 * q4 + 2],
                                            __uint_as_float(r[4 * q4 + 3]) + csum[c0 + 4 * q4 + 3]);
                }
            } else {
                // M = 64 accumulator: rows in lanes 0..15; the warp halves take column halves
                const int a = sp * 16 + (lane & 15);
                const int c0 = 32 * (lane >> 4);
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
                float4* o = reinterpret_cast<float4*>(rec + (size_t)a * D + c0);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    o[q4] = make_float4(__uint_as_float(r[4 * q4]) + csum[c0 + 4 * q4],
                                        __uint_as_float(r[4 * q4 + 1]) + csum[c0 + 4 * q4 + 1],
                                        __uint_as_float(r[4 * q4 + 2]) + csum[c0 + 4 * q4 + 2],
                                        __uint_as_float(r[4 * q4 + 3]) + csum[c0 + 4 * q4 + 3]);
            }
            tc_fence_before();
            named_bar(1, 128);  // `red` is reused by the next segment
        }
    }
    if constexpr (SCAN) {
        // Exclusive prefix of the head's block records across the cluster:
        // after the barrier (release / acquire at cluster scope, so every
        // record written above is visible) CTA r of the nc in the cluster
        // takes float4s [r*chunk, (r+1)*chunk) of the records, reads them
        // for every block in order (L2) and overwrites each with the sum over
        // the blocks before it, then writes the total. Each element has one
        // owner, so the in-place update needs no second barrier. Every thread
        // of every CTA reaches the barrier.
        cluster_sync();
        if (warp >= 2) {
            const int et = threadIdx.x - 64;
            const int nblk = w.nblk, bh = blockIdx.y, r = blockIdx.x, nc = gridDim.x;
            constexpr int E4 = (D * D + D) / 4;
            const int chunk = (E4 + nc - 1) / nc;
            float4* recs = reinterpret_cast<float4*>(part + (size_t)bh * nblk * REC);
            for (int f = r * chunk + et; f < min(E4, (r + 1) * chunk); f += 128) {
                float4 x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr)
                    if (rr < nblk) x[rr] = recs[(size_t)rr * (REC / 4) + f];
                float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    if (rr < nblk) {
                        recs[(size_t)rr * (REC / 4) + f] = run;
                        run.x += x[rr].x;
                        run.y += x[rr].y;
                        run.z += x[rr].z;
                        run.w += x[rr].w;
                    }
                }
                if (S_total != nullptr) {
                    const float t[4] = {run.x, run.y, run.z, run.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int idx = 4 * f + q;
                        if (idx < D * D) S_total[(size_t)bh * D * D + idx] = t[q];
                        else z_total[(size_t)bh * D + (idx - D * D)] = t[q];
                    }
                }
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

// Sums the partial records of each head in CTA order (deterministic).
__global__ void kv_reduce_balanced_kernel(const float* __restrict__ part, KvBalanced w, int D,
                                          float* __restrict__ S, float* __restrict__ z) {
    const int rec4 = (D * D + D) / 4;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const long long h = blockIdx.y;
    if (e >= rec4) {
        pdl_wait();
        return;
    }
    pdl_wait();
    const int c0 = cta_of(w, h * w.tph);
    const int c1 = cta_of(w, (h + 1) * w.tph - 1);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // eight record loads in flight at a time; the sum stays in CTA order
    for (int cb = c0; cb <= c1; cb += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = cb + u;
            if (c <= c1) {
                const long long j = h - range_lo(w.total, w.G, c) / w.tph;
                v[u] = reinterpret_cast<const float4*>(part + ((size_t)c * w.K + j) * (size_t)(rec4 * 4))[e];
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (cb + u <= c1) {
                acc.x += v[u].x;
                acc.y += v[u].y;
                acc.z += v[u].z;
                acc.w += v[u].w;
            }
        }
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
    // Q stages, S and z operands (x2), the output staging tile
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * TILE + 2 * BS + 2 * BZ + TILE + 8 * BARS + 16;
    static constexpr int PER_SM = D == 64 ? 2 : 1;     // CTAs an SM holds (TMEM and smem)
    static_assert(SMEM * PER_SM <= 227 * 1024, "shared memory");
};

template <int D, int PHI>
__global__ void __launch_bounds__(kThreads, RoCfg<D>::PER_SM)
tc_readout_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mOut,
                  const float* __restrict__ S, const float* __restrict__ z, int N, long long total,
                  int tph, int normalize, uint32_t* __restrict__ err) {
    using C = RoCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = align1024(smem_raw);
    uint8_t* bS = tiles + C::STAGES * C::TILE;
    uint8_t* bZ = bS + 2 * C::BS;
    uint8_t* stg = bZ + 2 * C::BZ;  // output tile, same layout as a Q tile
    uint64_t* full = reinterpret_cast<uint64_t*>(stg + C::TILE);
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
        cta_abort_reset();
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
        tma_prefetch_map(&mOut);
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
    // The TMA producer (warp 0) loads only the caller's Q, so it does not wait
    // for the previous kernel (the reduction of S, z) and fills the pipeline
    // while that kernel finishes; every other warp waits before it reads S, z.
    if (warp != 0) pdl_wait();

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
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
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
            if (ok && PHI != PHI_IDENTITY) {
                uint4* qt = reinterpret_cast<uint4*>(tiles + s * C::TILE);
#pragma unroll
                for (int i = 0; i < C::NB * 8; ++i) qt[et + 128 * i] = phi8<PHI>(qt[et + 128 * i]);
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
            // the staging tile is free once the previous tile's store has read it
            if (et == 0) bulk_wait_read0();
            named_bar(2, 128);
            const int r = sp * 32 + lane;  // row of the tile
            const float inv = normalize ? __frcp_rn(__uint_as_float(zr[0]) + __uint_as_float(zr[1])) : 1.0f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 8) {
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[c0 + e]) * inv;
                *reinterpret_cast<uint4*>(stg + (c0 / 64) * (kTile * 128) + sw128_off(r, c0 % 64)) = pack8(f);
            }
            fence_async_smem();
            named_bar(2, 128);
            if (et == 0 && ok) {
#pragma unroll
                for (int b = 0; b < C::NB; ++b)
                    tma_store_3d(&mOut, stg + b * (kTile * 128), b * 64, (int)(g % tph) * kTile, (int)(g / tph));
                bulk_commit();
            }
        };
        if (ntile > 0) transform(0);
        for (int it = 0; it < ntile; ++it) {
            if (it + 1 < ntile) transform(it + 1);
            epilogue(it);
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
cudaError_t launch_kv_phi(const Problem& p, const CUtensorMap& mk, const CUtensorMap& mv, const KvWork& w,
                          dim3 grid, float* part, uint32_t* err, cudaStream_t st) {
    constexpr size_t smem = KvCfg<D>::SMEM;
    cudaError_t e = ensure_smem<tc_kv_kernel<D, PHI>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_kv_kernel<D, PHI>, grid, dim3(kThreads), smem, st, mk, mv, p.N, w, part, err,
                      static_cast<float*>(nullptr), static_cast<float*>(nullptr));
}

// Blocks mode with the block-state scan inside: one cluster of nblk CTAs per head.
template <int D, int PHI>
cudaError_t launch_kv_scan(const Problem& p, const CUtensorMap& mk, const CUtensorMap& mv, const KvWork& w,
                           float* part, float* S_total, float* z_total, uint32_t* err, cudaStream_t st) {
    constexpr size_t smem = KvCfg<D, true>::SMEM;
    const cudaError_t e = ensure_smem<tc_kv_kernel<D, PHI, true>>(smem);
    if (e != cudaSuccess) return e;
    const unsigned nc = (unsigned)((w.nblk + w.bpc - 1) / w.bpc);  // CTAs of a head's cluster
    return launch_cluster_pdl(tc_kv_kernel<D, PHI, true>, dim3(nc, (unsigned)p.bh()), dim3(kThreads), smem, st, nc,
                              mk, mv, p.N, w, part, err, S_total, z_total);
}

// one kernel per feature map (see phi8)
template <int D>
cudaError_t launch_kv(const Problem& p, const void* k, const void* v, const KvWork& w, dim3 grid, float* part,
                      uint32_t* err, cudaStream_t st) {
    CUtensorMap mk, mv;
    cudaError_t e = make_map(&mk, k, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    switch (p.phi) {
        case PHI_RELU1: return launch_kv_phi<D, PHI_RELU1>(p, mk, mv, w, grid, part, err, st);
        case PHI_ELU1: return launch_kv_phi<D, PHI_ELU1>(p, mk, mv, w, grid, part, err, st);
        default: return launch_kv_phi<D, PHI_IDENTITY>(p, mk, mv, w, grid, part, err, st);
    }
}

template <int D, int PHI>
cudaError_t launch_readout_phi(const Problem& p, const CUtensorMap& mq, const CUtensorMap& mo, const float* S,
                               const float* z, uint32_t* err, cudaStream_t st) {
    constexpr size_t smem = RoCfg<D>::SMEM;
    cudaError_t e = ensure_smem<tc_readout_kernel<D, PHI>>(smem);
    if (e != cudaSuccess) return e;
    const int tph = (p.N + kTile - 1) / kTile;
    const long long total = p.bh() * tph;
    const int G = plan::balanced_ctas(total, device_sms(), RoCfg<D>::PER_SM);
    return launch_pdl(tc_readout_kernel<D, PHI>, dim3(G), dim3(kThreads), smem, st, mq, mo, S, z, p.N, total, tph,
                      p.normalize, err);
}

template <int D>
cudaError_t launch_readout(const Problem& p, const void* q, const float* S, const float* z, void* out,
                           uint32_t* err, cudaStream_t st) {
    CUtensorMap mq, mo;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mo, out, D, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1: return launch_readout_phi<D, PHI_RELU1>(p, mq, mo, S, z, err, st);
        case PHI_ELU1: return launch_readout_phi<D, PHI_ELU1>(p, mq, mo, S, z, err, st);
        default: return launch_readout_phi<D, PHI_IDENTITY>(p, mq, mo, S, z, err, st);
    }
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
    return launch_pdl(kv_reduce_balanced_kernel, dim3((rec4 + 127) / 128, (unsigned)p.bh()), dim3(128), 0, st,
                      part, w.b, p.d, S, z);
}

cudaError_t tc_reduce_records(const Problem& p, const KvBalanced& w, const float* part, float* S, float* z,
                              cudaStream_t st) {
    const int rec4 = (p.d * p.d + p.d) / 4;
    return launch_pdl(kv_reduce_balanced_kernel, dim3((rec4 + 127) / 128, (unsigned)p.bh()), dim3(128), 0, st, part,
                      w, p.d, S, z);
}

namespace {
// Clusters of cs CTAs with the scanning KV pass's threads and shared memory
// that the device holds at once (on a B200 at two CTAs per SM: 71 of 4, 33
// of 8, 14 of 16).
int cluster_capacity(int cs) { return max_active_clusters(cs, kThreads, KvCfg<64, true>::SMEM); }
// Blocks per CTA of the scanning KV pass: one while every head's cluster
// fits one wave, else two (half the CTAs, twice the tiles each); 0 when
// neither fits (the separate scan kernel is used then).
int kv_scan_bpc(const Problem& p, int nblk) {
    for (int bpc = 1; bpc <= 2; ++bpc)
        if (p.bh() <= cluster_capacity((nblk + bpc - 1) / bpc)) return bpc;
    return 0;
}
}  // namespace

bool tc_kv_scan_supported(const Problem& p, int block_tokens, int nblk) {
    // one cluster per head (at most 16 blocks), all clusters in one wave
    return tc_supported(p) && p.d == 64 && block_tokens % kTile == 0 && nblk >= 1 && nblk <= 16 &&
           kv_scan_bpc(p, nblk) > 0;
}

cudaError_t tc_kv_blocks_scan(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                              float* S_total, float* z_total, uint32_t* err, cudaStream_t st) {
    if (!tc_kv_scan_supported(p, block_tokens, nblk)) return cudaErrorInvalidValue;
    KvWork w{};
    w.balanced = 0;
    w.block_tokens = block_tokens;
    w.nblk = nblk;
    w.bpc = kv_scan_bpc(p, nblk);
    CUtensorMap mk, mv;
    cudaError_t e = make_map(&mk, k, 64, p.N, p.bh(), kTile);
    if (e == cudaSuccess) e = make_map(&mv, v, 64, p.N, p.bh(), kTile);
    if (e != cudaSuccess) return e;
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1: return launch_kv_scan<64, PHI_RELU1>(p, mk, mv, w, part, S_total, z_total, err, st);
        case PHI_ELU1: return launch_kv_scan<64, PHI_ELU1>(p, mk, mv, w, part, S_total, z_total, err, st);
        default: return launch_kv_scan<64, PHI_IDENTITY>(p, mk, mv, w, part, S_total, z_total, err, st);
    }
}

cudaError_t tc_kv_blocks(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                         uint32_t* err, cudaStream_t st, int nform) {
    if (block_tokens % kTile != 0) return cudaErrorInvalidValue;
    if (nform < 0) nform = nblk;
    if (nform > nblk) return cudaErrorInvalidValue;
    if (nform == 0) return cudaSuccess;
    KvWork w{};
    w.balanced = 0;
    w.block_tokens = block_tokens;
    w.nblk = nblk;
    w.bpc = 1;
    const dim3 grid(nform, (unsigned)p.bh());  // records keep the stride of nblk blocks per head
    return p.d == 64 ? launch_kv<64>(p, k, v, w, grid, part, err, st)
                     : launch_kv<128>(p, k, v, w, grid, part, err, st);
}

cudaError_t tc_readout(const Problem& p, const void* q, const float* S, const float* z, void* out, uint32_t* err,
                       cudaStream_t st) {
    return p.d == 64 ? launch_readout<64>(p, q, S, z, out, err, st)
                     : launch_readout<128>(p, q, S, z, out, err, st);
}

}  // namespace la
