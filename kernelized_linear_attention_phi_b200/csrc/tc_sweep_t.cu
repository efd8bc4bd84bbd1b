// Chunked causal / prefix-mask attention for d = 128 on tcgen05 tensor cores
// (bf16), with the running state kept transposed.
//
// The d = 64 kernel (tc_sweep.cu) multiplies phi(Q) by the state with the
// queries as the M dimension; at d = 128 with 64-token chunks that puts the
// two large products (phi(Q) S_prev and P~ V) on half-rate M = 64
// instructions and needs a 64 KB shared-memory copy of S_prev. Here the state
// is held as S^T (d_v lanes x d_k columns) and the outputs as O^T, so both
// products have M = d_v = 128:
//   S^T += V_c^T phi(K_c)                  A = V^T (smem), B = phi(K) (smem)
//   O^T  = S_prev^T phi(Q)^T               A = S_prev^T as bf16 in TMEM
//   O^T += V_c^T P~^T                      A = V^T,  B = P~ (smem)
// and S_prev^T never leaves TMEM (fp32 -> bf16 pairs, lane for lane). The
// normaliser rides along with the score product: the K tile of a chunk gets
// 16 extra rows, row 64 = bf16(z_prev), row 65 = the rounding remainder, the
// rest zero, so P = phi(Q) [phi(K_c); z_hi; z_lo; 0]^T carries phi(Q_i).z_prev
// in its columns 64 and 65. z itself is summed on the CUDA cores from the
// transformed K tiles.
//
// Warp roles (320 threads) as in the d = 64 kernel: warp 0 TMA (with the
// gathered query rows and their row table for the prefix mask), warp 1 MMA +
// TMEM, warps 2-5 "prep" (phi on K / Q, z, S^T -> bf16), warps 6-9 "mask"
// (P~, denominators, epilogue). Three pipeline stages; P, O^T and
// P~ are double-buffered by tile parity, and the MMA warp issues a tile's
// O^T += V^T P~^T only after the next tile's P and O^T, so the tensor core
// has work while the mask warps turn P into P~.

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

template <bool GATHER>
struct StCfg {
    static constexpr int D = 128, C = 64, NB = 2;
    static constexpr int BOX = C * 128;               // one 64-row x 64-column box (8 KB)
    static constexpr int KBOX = (C + 16) * 128;       // K box + 16 rows (z_hi, z_lo, zeros)
    static constexpr int TILE = NB * BOX;             // one [C x D] bf16 tile (16 KB)
    static constexpr int OFF_K = GATHER ? 0 : TILE;   // stage: (Q,) K', V
    static constexpr int OFF_V = OFF_K + NB * KBOX;
    static constexpr int STAGE = OFF_V + TILE;
    static constexpr uint32_t TX = (GATHER ? 2 : 3) * TILE;  // bytes TMA brings per stage
    static constexpr int STAGES = 3;
    static constexpr int PT = C * C * 2;              // P~ [query][key], K-major (x2)
    static constexpr int STG = TILE;                  // output staging tile
    static constexpr int QG = GATHER ? 2 * TILE : 0;  // gathered queries (x2)
    static constexpr int ROWS = GATHER ? 2 * 2 * C * 4 : 0;
    static constexpr int OROWS = GATHER ? 2 * C * 4 : 0;  // output rows of a gathered tile (x2)
    static constexpr int RED = 2 * 4 * D * 4;         // column-sum partials [parity][warp][d_k]
    static constexpr int INV = C * 4;                 // 1 / den per query row
    static constexpr int NBAR = 2 * STAGES + 2 + 6 * 2;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * PT + STG + QG + ROWS + OROWS + RED + INV +
                                   8 * NBAR + 16;
    // TMEM columns
    static constexpr int COL_S = 0;      // S^T fp32 [d_v lanes][d_k]
    static constexpr int COL_SB = 128;   // S_prev^T bf16 pairs [d_v lanes][d_k / 2], 2 x 64
    static constexpr int COL_P = 256;    // P (M = 64) [query][C + 16]; slot 1 in lanes 16..31
    static constexpr int COL_O = 384;    // O^T fp32 [d_v lanes][query], 2 x 64
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 320;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && KBOX % 1024 == 0, "1024-byte aligned operand tiles");
};

template <bool GATHER, int PHI>
__global__ void __launch_bounds__(StCfg<GATHER>::THREADS, 1)
tc_sweep_t_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                  const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mOut,
                  const float* __restrict__ prefix, int H, int N,
                  int block_tokens, int nblk, const int32_t* __restrict__ perm,
                  const int32_t* __restrict__ bin_start, const int32_t* __restrict__ msort, int nbins,
                  int normalize, int raw_prefix, __nv_bfloat16* __restrict__ out, uint32_t* __restrict__ err) {
    using CF = StCfg<GATHER>;
    constexpr int D = CF::D, C = CF::C;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* pt = stages + CF::STAGES * CF::STAGE;
    uint8_t* stg = pt + 2 * CF::PT;
    uint8_t* qg = stg + CF::STG;
    int* rows = reinterpret_cast<int*>(qg + CF::QG);  // [slot][srow C | slim C]
    int* orows = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(rows) + CF::ROWS);  // [slot][C]
    float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(orows) + CF::OROWS);
    float* inv = red + 2 * 4 * D;
    uint64_t* full = reinterpret_cast<uint64_t*>(inv + C);
    uint64_t* empty = full + CF::STAGES;
    uint64_t* bprep = empty + CF::STAGES;  // K', Q transformed and S_prev^T in TMEM
    uint64_t* bsdone = bprep + 1;          // S^T update of the chunk done
    // Per-tile barriers, per slot (tile t uses slot t % 2, phase t / 2): P
    // ready, P~ written (P read), O^T ready, O^T read, queries transformed,
    // and (prefix mask) query rows landed with their row table.
    uint64_t* bpfull = bsdone + 1;
    uint64_t* bptready = bpfull + 2;
    uint64_t* bofull = bptready + 2;
    uint64_t* bofree = bofull + 2;
    uint64_t* bqready = bofree + 2;
    uint64_t* qfull = bqready + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfull + 2);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    const int c_end = (GATHER && blk == nblk - 1) ? nbins : min(nchunks, c_begin + block_tokens / C);
    const int nci = c_end - c_begin;
    constexpr bool mapped = PHI != PHI_IDENTITY;  // phi applied to Q and K tiles
    const size_t hoff = (size_t)bh * N * D;

    auto q_tiles = [&](int c) -> int {
        if (!GATHER) return c < nchunks ? 1 : 0;
        const int cnt = bin_start[(size_t)b * (nbins + 1) + c + 1] - bin_start[(size_t)b * (nbins + 1) + c];
        return (cnt + C - 1) / C;
    };

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(bprep, 128);
        mbar_init(bsdone, 1);
        for (int j = 0; j < 2; ++j) {
            mbar_init(bpfull + j, 1);
            mbar_init(bptready + j, 128);
            mbar_init(bofull + j, 1);
            mbar_init(bofree + j, 128);
            mbar_init(bqready + j, 128);
            mbar_init(qfull + j, 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, CF::TMEM_COLS);
    if (threadIdx.x == 0) {
        tma_prefetch_map(&mQ);
        if (!GATHER) tma_prefetch_map(&mOut);
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The TMA producer (warp 0) first loads only the caller's inputs, so it
    // fills the pipeline without waiting for the previous kernel of the call;
    // every other warp waits before it reads what that kernel wrote.
    if (warp != 0) pdl_wait();

    if (warp == 0) {
        // ---------------- TMA producer (whole warp) ----------------
        auto load_chunk = [&](int ci) {
            const int s = ci % CF::STAGES;
            if (lane == 0) {
                mbar_arrive_expect_tx(full + s, CF::TX);
                uint8_t* st = stages + s * CF::STAGE;
                const int row = (c_begin + ci) * C;
#pragma unroll
                for (int bx = 0; bx < CF::NB; ++bx) {
                    if (!GATHER) tma_load_3d(st + bx * CF::BOX, &mQ, full + s, bx * 64, row, bh);
                    tma_load_3d(st + CF::OFF_K + bx * CF::KBOX, &mK, full + s, bx * 64, row, bh);
                    tma_load_3d(st + CF::OFF_V + bx * CF::BOX, &mV, full + s, bx * 64, row, bh);
                }
            }
        };
        int nld = min(nci, CF::STAGES);
        for (int ci = 0; ci < nld; ++ci) load_chunk(ci);
        // the bin tables below come from an earlier kernel of the call
        if (GATHER) pdl_wait();
        bool ok = true;
        int tq = 0;
        for (int ci = 0; ci < nci && ok; ++ci) {
            if (ci >= CF::STAGES) {
                const int s = ci % CF::STAGES, u = ci / CF::STAGES;
                ok = __all_sync(0xffffffffu, mbar_wait(empty + s, (u - 1) & 1, err));
                if (!ok) break;
                load_chunk(ci);
                nld = ci + 1;
            }
            if (GATHER) {
                const int c = c_begin + ci;
                const int qbase = bin_start[(size_t)b * (nbins + 1) + c];
                const int qend = bin_start[(size_t)b * (nbins + 1) + c + 1];
                for (int t = 0; qbase + t * C < qend; ++t, ++tq) {
                    constexpr int R = C / 32;  // rows of the tile per lane
                    const int slot = tq & 1;
                    int tok[R], lim[R];
#pragma unroll
                    for (int e = 0; e < R; ++e) {
                        const int idx = qbase + t * C + R * lane + e;
                        tok[e] = idx < qend ? perm[(size_t)b * N + idx] : -1;
                        lim[e] = idx < qend ? msort[(size_t)b * N + idx] - c * C : -1;
                    }
                    // the slot's previous tile has been read out (and its row table with it)
                    if (tq >= 2) ok = __all_sync(0xffffffffu, mbar_wait(bofree + slot, ((tq >> 1) - 1) & 1, err));
                    if (!ok) break;
                    int* srow = rows + slot * 2 * C;
#pragma unroll
                    for (int e = 0; e < R; ++e) {
                        srow[R * lane + e] = tok[e];
                        srow[C + R * lane + e] = lim[e];
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_expect_tx(qfull + slot, CF::TILE);
                    __syncwarp();
                    gather_tile<C, CF::NB>(qg + slot * CF::TILE, &mQ, qfull + slot, bh * N, tok, lane);
                }
            }
        }
        // drain: the loads still in flight land before the CTA exits
        if (lane == 0) {
            for (int c2 = max(0, nld - CF::STAGES); c2 < nld; ++c2)
                mbar_wait(full + c2 % CF::STAGES, (c2 / CF::STAGES) & 1, err, false);
            for (int t2 = max(0, tq - 2); t2 < tq; ++t2) mbar_wait(qfull + (t2 & 1), (t2 >> 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const int NP = normalize ? C + 16 : C;
            const uint32_t idP = idesc_bf16(C, NP, false, false);     // P = Q [K; z]^T
            constexpr uint32_t idS = idesc_bf16(D, D, true, true);    // S^T += V^T K
            constexpr uint32_t idO = idesc_bf16(D, C, false, false);  // O^T = S_prev^T Q^T
            constexpr uint32_t idV = idesc_bf16(D, C, true, false);   // O^T += V^T P~^T
            const uint32_t pta = smem_u32(pt);
            bool ok = true;
            // the tile whose O^T += V^T P~^T is still to be issued
            int pend = -1, pend_stage = -1;
            uint32_t pend_vt = 0;
            auto flush = [&]() {
                if (pend < 0 || !ok) return;
                const int j = pend & 1, k = pend >> 1;
                ok = mbar_wait(bptready + j, k & 1, err);
                if (!ok) return;
                tc_fence_after();
                const uint32_t ptj = pta + j * CF::PT;
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + CF::COL_O + j * C, sdesc(pend_vt + kk * 2048, CF::BOX, 1024),
                             sdesc(ptj + kk * 32, 16, 1024), idV, 1u);
                mma_commit(bofull + j);
                if (pend_stage >= 0) mma_commit(empty + pend_stage);
                pend = -1;
            };
            int tq = 0;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t st = smem_u32(stages + s * CF::STAGE);
                const uint32_t kt = st + CF::OFF_K, vt = st + CF::OFF_V;
                flush();
                if (!ok) break;
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + CF::COL_S, sdesc(vt + kk * 2048, CF::BOX, 1024),
                             sdesc(kt + kk * 2048, CF::KBOX, 1024), idS, 1u);
                mma_commit(bsdone);
                const uint32_t sb = tmem + CF::COL_SB + (ci & 1) * 64;
                const int ntq = q_tiles(c_begin + ci);
                for (int t = 0; t < ntq && ok; ++t, ++tq) {
                    const int j = tq & 1, k = tq >> 1;
                    const uint32_t qt = GATHER ? smem_u32(qg + j * CF::TILE) : st;
                    if (GATHER) ok = mbar_wait(bqready + j, k & 1, err);
                    if (!ok) break;
                    tc_fence_after();
                    // P[j] was read two tiles ago (that tile's P~ was waited for in its flush)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16(tmem + CF::COL_P + j * (16u << 16),
                                 sdesc(qt + (kk / 4) * CF::BOX + (kk % 4) * 32, 16, 1024),
                                 sdesc(kt + (kk / 4) * CF::KBOX + (kk % 4) * 32, 16, 1024), idP, kk > 0);
                    mma_commit(bpfull + j);
                    if (k > 0) ok = mbar_wait(bofree + j, (k - 1) & 1, err);  // O^T[j] read two tiles ago
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ts(tmem + CF::COL_O + j * C, sb + kk * 8,
                                    sdesc(qt + (kk / 4) * CF::BOX + (kk % 4) * 32, 16, 1024), idO, kk > 0);
                    if (t > 0) flush();
                    pend = tq;
                    pend_vt = vt;
                    pend_stage = t == ntq - 1 ? s : -1;
                }
                if (ntq == 0) mma_commit(empty + s);
            }
            flush();
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int a = sp * 32 + lane;  // the S^T row (d_v index) this thread owns in TMEM
        // the block's prefix: its record of the exclusive block scan, or with
        // raw_prefix the records of the blocks before it (their own states),
        // summed here in block order (the order the scan adds them in)
        constexpr size_t kRec = (size_t)D * D + D;
        const float* pre = prefix + ((size_t)bh * nblk + (raw_prefix ? 0 : blk)) * kRec;
        const int npre = raw_prefix ? blk : 1;
        // rows 66..79 of every extended K box stay zero (TMA writes rows 0..63)
        for (int x = et; x < CF::STAGES * CF::NB * 14 * 8; x += 128) {
            const int s = x / (CF::NB * 112), bx = (x / 112) % CF::NB, r = 66 + (x % 112) / 8, q16 = x % 8;
            *reinterpret_cast<uint4*>(stages + s * CF::STAGE + CF::OFF_K + bx * CF::KBOX + r * 128 + q16 * 16) =
                make_uint4(0, 0, 0, 0);
        }
        // seed S^T with the block's prefix record (S stored [d_k][d_v]); the
        // loads of four records are in flight at a time (one L2 round trip
        // per four records, not per record), the sum keeps block order
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
            float f[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) f[e] = 0.f;
            int rb = 0;
#pragma unroll 1
            for (; rb + 4 <= npre; rb += 4) {
                float t[4][16];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 16; ++e) t[j][e] = pre[(rb + j) * kRec + (size_t)(c0 + e) * D + a];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 16; ++e) f[e] += t[j][e];
            }
#pragma unroll 1
            for (; rb < npre; ++rb) {
#pragma unroll
                for (int e = 0; e < 16; ++e) f[e] += pre[rb * kRec + (size_t)(c0 + e) * D + a];
            }
            uint32_t r[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(f[e]);
            tmem_st16(tmem + CF::COL_S + lane_base + c0, r);
        }
        tmem_st_wait();
        float zp = 0.f;  // z_prev[d_k = et]
        if (normalize)
            for (int rb = 0; rb < npre; ++rb) zp += pre[rb * kRec + (size_t)D * D + et];
        // column group (of 8) of the K chunks this thread transforms: the
        // 128-byte swizzle maps 16-byte chunk (lane & 7) of its rows (all with
        // the same row & 7) to logical columns 8 * g .. 8 * g + 7
        const int g = (lane & 7) ^ ((et >> 3) & 7);
        int tq = 0;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
            uint8_t* st = stages + s * CF::STAGE;
            uint8_t* kt = st + CF::OFF_K;
            mbar_wait(full + s, u & 1, err);
            if (normalize) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(zp);
                const __nv_bfloat16 lo = __float2bfloat16_rn(zp - __bfloat162float(hi));
                uint8_t* kb = kt + (et / 64) * CF::KBOX;
                *reinterpret_cast<__nv_bfloat16*>(kb + sw128_off(C, et % 64)) = hi;
                *reinterpret_cast<__nv_bfloat16*>(kb + sw128_off(C + 1, et % 64)) = lo;
            }
            float* rp = red + (ci & 1) * 4 * D;
#pragma unroll
            for (int bx = 0; bx < CF::NB; ++bx) {
                float cs[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) cs[e] = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int w = et + 128 * i;  // 16-byte chunk within the box
                    const int r = w >> 3;
                    uint4* kp = reinterpret_cast<uint4*>(kt + bx * CF::KBOX + w * 16);
                    uint4 x = *kp;
                    if (r < kvalid) {
                        if (mapped) x = phi8<PHI>(x);
                    } else {
                        x = make_uint4(0, 0, 0, 0);
                    }
                    *kp = x;
                    if (normalize) {
                        float f[8];
                        unpack8(x, f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) cs[e] += f[e];
                    }
                    if (!GATHER && mapped) {
                        uint4* qp = reinterpret_cast<uint4*>(st + bx * CF::BOX + w * 16);
                        *qp = phi8<PHI>(*qp);
                    }
                }
                if (normalize) {
                    // lanes l, l^9, l^18, l^27 hold the same column group g
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 9);
                        cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 18);
                    }
                    if (lane < 8) {
                        float4* dst = reinterpret_cast<float4*>(rp + (warp - 2) * D + bx * 64 + g * 8);
                        dst[0] = make_float4(cs[0], cs[1], cs[2], cs[3]);
                        dst[1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
                    }
                }
            }
            if (normalize) {
                named_bar(2, 128);
                zp += (rp[et] + rp[D + et]) + (rp[2 * D + et] + rp[3 * D + et]);
            }
            if (ci > 0) {
                mbar_wait(bsdone, (ci - 1) & 1, err);
                tc_fence_after();
            }
            // S_prev^T -> bf16 pairs in TMEM, lane for lane
            const uint32_t sb = tmem + CF::COL_SB + (ci & 1) * 64 + lane_base;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t r[32];
                tmem_ld16(tmem + CF::COL_S + lane_base + 32 * h, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16(tmem + CF::COL_S + lane_base + 32 * h + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) w[e] = pack_bf16(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
                tmem_st16(sb + 16 * h, w);
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);

            if (GATHER) {
                // the gathered query rows of the chunk's tiles: phi in place
                const int ntq = q_tiles(c);
                for (int t = 0; t < ntq; ++t, ++tq) {
                    const int slot = tq & 1;
                    mbar_wait(qfull + slot, (tq >> 1) & 1, err);
                    if (mapped) {
                        constexpr int NL = C * D / 8 / 128;
                        uint4* q = reinterpret_cast<uint4*>(qg + slot * CF::TILE);
                        uint4 w[NL];
#pragma unroll
                        for (int j = 0; j < NL; ++j) w[j] = q[et + 128 * j];
#pragma unroll
                        for (int j = 0; j < NL; ++j) q[et + 128 * j] = phi8<PHI>(w[j]);
                        fence_async_smem();
                    }
                    mbar_arrive(bqready + slot);
                }
            }
        }
    } else {
        // ---------------- mask + epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int i = sp * 16 + (lane & 15);  // P row (query) of this thread: M = 64 layout
        const int half = lane >= 16 ? 1 : 0;  // the two warp halves take the two column halves
        const int et2 = threadIdx.x - 192;
        // No early exit in this warpgroup (named barrier 3); a failed wait
        // only suppresses the output stores.
        bool ok = true;
        int tq = 0;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int ntq = q_tiles(c);
            for (int t = 0; t < ntq; ++t, ++tq) {
                const int slot = tq & 1, use = tq >> 1;
                const uint32_t lane_s = lane_base + static_cast<uint32_t>(slot) * (16u << 16);
                uint8_t* pts = pt + slot * CF::PT;
                ok = mbar_wait(bpfull + slot, use & 1, err) && ok;
                // the row table of a gathered tile (written by the TMA warp)
                if (GATHER) ok = mbar_wait(qfull + slot, use & 1, err) && ok;
                tc_fence_after();
                const int* srow = rows + slot * 2 * C;
                const int lim = GATHER ? srow[C + i] : i;
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + CF::COL_P + lane_s, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + CF::COL_P + lane_s + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                uint32_t zq = 0;
                if (normalize) tmem_ld1x2<1>(tmem + CF::COL_P + lane_s + C, zq);
                tmem_ld_wait();
                float rs = 0.f;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * half + 8 * gq + e;
                        f[e] = j <= lim ? __uint_as_float(r[8 * gq + e]) : 0.f;
                        rs += f[e];
                    }
                    *reinterpret_cast<uint4*>(pts + sw128_off(i, 32 * half + 8 * gq)) = pack8(f);
                }
                if (normalize) {
                    rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                    float qz = __uint_as_float(zq);  // phi(Q_i).z_hi (lanes < 16), .z_lo (lanes >= 16)
                    qz += __shfl_xor_sync(0xffffffffu, qz, 16);
                    if (lane < 16) inv[i] = __frcp_rn(rs + qz);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bptready + slot);
                // epilogue: this thread's d_v column of the tile's output rows
                ok = ok && mbar_wait(bofull + slot, use & 1, err);
                tc_fence_after();
                // gathered rows: keep the tile's output rows past the release
                // of the row table (bofree below)
                if (GATHER && et2 < C) orows[slot * C + et2] = srow[et2];
                if (!GATHER && et2 == 0) bulk_wait_read0();  // the previous tile's store has read stg
                named_bar(3, 128);  // also: the previous copy-out is done, inv[] is written
                // O^T rows (d_v) a0 .. a0 + 15 per lane half, 16 columns (queries)
                // at a time: the 16x256b TMEM shape hands each lane two rows x two
                // adjacent columns, which is the fragment stmatrix .trans stores as
                // 8 x 8 blocks with the queries as rows (16 bytes of d_v each).
                const int mi = lane >> 3, mj = lane & 7;  // the block, and its row, this lane addresses
                const int q2 = 2 * (lane & 3);           // this lane's first column within 8
                const uint32_t stg_u = smem_u32(stg);
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const int a0 = sp * 32 + 16 * hl;
                    uint32_t o[32];
                    tmem_ld16x256_x8(tmem + CF::COL_O + slot * C + (static_cast<uint32_t>(a0) << 16), o);
                    tmem_ld_wait();
                    if (hl == 1) {
                        tc_fence_before();
                        mbar_arrive(bofree + slot);  // O^T[slot] read (and, gathered, the row table)
                    }
                    const uint32_t box = stg_u + (a0 / 64) * CF::BOX;
                    const int ch = (a0 % 64) / 8 + (mi & 1);  // 16-byte column chunk of the addressed block
#pragma unroll
                    for (int cb = 0; cb < C; cb += 16) {
                        const float2 i0 = normalize ? *reinterpret_cast<const float2*>(inv + cb + q2)
                                                    : make_float2(1.f, 1.f);
                        const float2 i1 = normalize ? *reinterpret_cast<const float2*>(inv + cb + 8 + q2)
                                                    : make_float2(1.f, 1.f);
                        const uint32_t* r = o + (cb / 8) * 4;
                        const uint32_t p0 = pack_bf16(__uint_as_float(r[0]) * i0.x, __uint_as_float(r[1]) * i0.y);
                        const uint32_t p1 = pack_bf16(__uint_as_float(r[2]) * i0.x, __uint_as_float(r[3]) * i0.y);
                        const uint32_t p2 = pack_bf16(__uint_as_float(r[4]) * i1.x, __uint_as_float(r[5]) * i1.y);
                        const uint32_t p3 = pack_bf16(__uint_as_float(r[6]) * i1.x, __uint_as_float(r[7]) * i1.y);
                        const uint32_t row = cb + 8 * (mi >> 1) + mj;
                        stmatrix_x4_trans(box + row * 128u + ((static_cast<uint32_t>(ch) ^ (row & 7u)) << 4), p0, p1,
                                          p2, p3);
                    }
                }
                fence_async_smem();
                named_bar(3, 128);
                if (!GATHER) {
                    if (et2 == 0 && ok) {
#pragma unroll
                        for (int bx = 0; bx < CF::NB; ++bx) tma_store_3d(&mOut, stg + bx * CF::BOX, bx * 64, c * C, bh);
                        bulk_commit();
                    }
                } else {
                    // a full row per 16 consecutive threads
#pragma unroll
                    for (int j = 0; j < C * D / 8 / 128; ++j) {
                        const int p = et2 + 128 * j;
                        const int rr = p / (D / 8), cc = (p % (D / 8)) * 8;
                        const int dst = orows[slot * C + rr];
                        if (ok && dst >= 0)
                            *reinterpret_cast<uint4*>(out + hoff + (size_t)dst * D + cc) =
                                *reinterpret_cast<const uint4*>(stg + (cc / 64) * CF::BOX + sw128_off(rr, cc % 64));
                    }
                }
            }
        }
    }
    if (!GATHER && threadIdx.x == 192) bulk_wait0();  // the output stores have landed
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CF::TMEM_COLS);
    }
}

template <bool GATHER, int PHI>
cudaError_t launch_t(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                     int block_tokens, int nblk, const int32_t* perm, const int32_t* bins, const int32_t* msort,
                     int nbins, int raw_prefix, void* out, uint32_t* err, cudaStream_t st) {
    using CF = StCfg<GATHER>;
    if (p.d != CF::D || block_tokens % CF::C != 0) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    // gathered queries: a 2-D row map for tile::gather4
    cudaError_t e = GATHER ? make_row_map(&mq, q, CF::D, p.bh() * p.N) : make_map(&mq, q, CF::D, p.N, p.bh(), CF::C);
    if (e == cudaSuccess) e = make_map(&mk, k, CF::D, p.N, p.bh(), CF::C);
    if (e == cudaSuccess) e = make_map(&mv, v, CF::D, p.N, p.bh(), CF::C);
    if (e == cudaSuccess) e = make_map(&mo, out, CF::D, p.N, p.bh(), CF::C);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_sweep_t_kernel<GATHER, PHI>>(CF::SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid(nblk, (unsigned)p.bh());
    return launch_pdl(tc_sweep_t_kernel<GATHER, PHI>, grid, dim3(CF::THREADS), CF::SMEM, st, mq, mk, mv, mo,
                      prefix, p.H, p.N, block_tokens, nblk, perm, bins, msort, nbins, p.normalize, raw_prefix,
                      static_cast<__nv_bfloat16*>(out), err);
}

// one kernel per feature map (see phi8)
template <bool GATHER>
cudaError_t launch_phi(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                       int block_tokens, int nblk, const int32_t* perm, const int32_t* bins, const int32_t* msort,
                       int nbins, int raw_prefix, void* out, uint32_t* err, cudaStream_t st) {
    switch (p.phi) {
        case PHI_RELU1:
            return launch_t<GATHER, PHI_RELU1>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins,
                                               raw_prefix, out, err, st);
        case PHI_ELU1:
            return launch_t<GATHER, PHI_ELU1>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins,
                                              raw_prefix, out, err, st);
        default:
            return launch_t<GATHER, PHI_IDENTITY>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort,
                                                  nbins, raw_prefix, out, err, st);
    }
}

}  // namespace

cudaError_t tc_chunked_t(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                         int block_tokens, int nblk, const int32_t* perm, const int32_t* bins,
                         const int32_t* msort, int nbins, void* out, uint32_t* err, cudaStream_t st,
                         bool raw_prefix) {
    if (perm != nullptr)
        return launch_phi<true>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins, raw_prefix ? 1 : 0,
                                out, err, st);
    return launch_phi<false>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins, raw_prefix ? 1 : 0, out,
                             err, st);
}

}  // namespace la
