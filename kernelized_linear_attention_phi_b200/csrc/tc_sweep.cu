// Chunked causal / prefix-mask attention on tcgen05 tensor cores (bf16).
// See the comment above the kernel for the algorithm and the warp roles.

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

// ---------------------------------------------------------------------------
// Chunked causal / prefix-mask outputs of one block
// ---------------------------------------------------------------------------
// The block's chunks are swept in order with the running state of all
// earlier keys: S in TMEM (fp32, M = d_k rows) and z in the prep warps'
// registers (fp32, one entry per thread), both seeded from the block's
// prefix record. For chunk c (C keys) and each tile of up to C queries
// answered there:
//   S_prev, z_prev -> bf16 operands (z as hi + lo rows)      [prep warps]
//   z += column sums of phi(K_c) (fp32, CUDA cores)            [prep warps]
//   S += phi(K_c)^T V_c                                        [MMA]
//   P  = phi(Q) phi(K_c)^T                                     [MMA, M = C]
//   P~ = P with keys j > lim_i zeroed, bf16; den_i = rowsum   [mask warps]
//   O  = phi(Q) S_prev + P~ V_c ; Oz = phi(Q) z_prev           [MMA]
//   out_i = O_i / (den_i + Oz_i)                               [mask warps]
// Causal: the queries of chunk c are its own tokens, lim_i = i - cC.
// Prefix mask: the queries of bin c (floor((m_i+1)/C) = c) are gathered
// rows, lim_i = m_i - cC in [-1, C-2].
//
// Warp roles (320 threads): warp 0 TMA (K / V (/ Q) chunks; for the prefix
// mask also each tile of gathered query rows, by tile::gather4 through a 2-D
// row map of Q, and the tile's row table), warp 1 MMA + TMEM, warps 2-5
// "prep" (phi on the K / Q tiles, state -> operands), warps 6-9 "mask" (P~,
// epilogue). Prep runs one chunk ahead of mask; the S / z operands are
// double-buffered. Gathered query tiles sit in a ring of QS slots of their
// own, so that each tile's gather (scattered rows, the longest load of the
// kernel) is issued QS - 1 tiles before its use. The per-tile accumulators
// (P, O, Oz) and the P~ operand are double-buffered by tile parity ("slot"),
// so the tensor core starts tile t+1 while the mask warps finish tile t: with
// 64-row chunks (M = 64 accumulators, which use TMEM lanes 0..15 of each
// sub-partition) slot 1 lives in lanes 16..31 of the same columns, with
// 128-row chunks in separate columns.
template <int D, int C, bool GATHER>
struct SwCfg {
    static constexpr int NB = D / 64;
    static constexpr int TILE = C * D * 2;           // one [C x D] bf16 tile
    static constexpr int NT = GATHER ? 2 : 3;        // tiles per stage: (Q,) K, V
    static constexpr int STAGES = 2;
    static constexpr int STAGE = NT * TILE;
    static constexpr int PT = C * C * 2;             // P~, K-major (x2)
    static constexpr int B3 = D * D * 2;             // S_prev, MN-major (x2)
    static constexpr int BZ = 16 * D * 2;            // z_hi, z_lo, 14 zero rows; K-major (x2)
    static constexpr int RED = 2 * 4 * D * 4;        // z column-sum partials [parity][warp][d]
    static constexpr int QS = GATHER ? 3 : 1;        // gathered query slots
    static constexpr int QG = GATHER ? QS * TILE : 0;
    static constexpr int ROWS = GATHER ? QS * 2 * C * 4 : 0;  // token / limit per row, per query slot
    static constexpr int STG = TILE;                 // output staging tile
    // TMEM columns: S, then P, O, Oz (two slots each; see above)
    static constexpr int SLOTC = C == 64 ? 1 : 2;    // column copies per slot pair
    static constexpr int COL_S = 0, COL_P = D, COL_O = COL_P + SLOTC * C, COL_OZ = COL_O + SLOTC * D,
                         COL_END = COL_OZ + SLOTC * 16;
    static constexpr uint32_t TMEM_COLS = COL_END <= 256 ? 256u : 512u;
    static_assert(COL_END <= 512, "TMEM");
    static constexpr int NBAR = 2 * STAGES + 2 + 4 * 2 + 3 * QS;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * PT + 2 * B3 + 2 * BZ + QG + STG + ROWS +
                                   RED + 8 * NBAR + 16;
    // TMEM address offsets of slot j for P, O and Oz
    __device__ static constexpr uint32_t p_slot(int j) { return C == 64 ? (uint32_t)j * (16u << 16) : (uint32_t)j * C; }
    __device__ static constexpr uint32_t o_slot(int j) { return C == 64 ? (uint32_t)j * (16u << 16) : (uint32_t)j * D; }
    __device__ static constexpr uint32_t oz_slot(int j) { return C == 64 ? (uint32_t)j * (16u << 16) : (uint32_t)j * 16; }
    static constexpr int THREADS = 320;
    static constexpr int MIN_BLOCKS = (D == 64 && C == 64) ? 2 : 1;
    static_assert(C == 64 || C == 128, "chunk");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    // two resident CTAs per SM: 228 KiB per SM, 1 KiB reserved per CTA
    static_assert(MIN_BLOCKS == 1 || MIN_BLOCKS * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
};

template <int D, int C, bool GATHER, int PHI>
__global__ void __launch_bounds__(SwCfg<D, C, GATHER>::THREADS, SwCfg<D, C, GATHER>::MIN_BLOCKS)
tc_sweep_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mOut,
                const float* __restrict__ prefix, int H, int N, int block_tokens, int nblk,
                const int32_t* __restrict__ perm, const int32_t* __restrict__ bin_start,
                const int32_t* __restrict__ msort, int nbins, int normalize,
                __nv_bfloat16* __restrict__ out, uint32_t* __restrict__ err) {
    using CF = SwCfg<D, C, GATHER>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* pt = stages + CF::STAGES * CF::STAGE;
    uint8_t* b3 = pt + 2 * CF::PT;
    uint8_t* bz = b3 + 2 * CF::B3;
    uint8_t* qg = bz + 2 * CF::BZ;
    uint8_t* stg = qg + CF::QG;
    int* rows = reinterpret_cast<int*>(stg + CF::STG);  // [query slot][srow C | slim C]
    float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(rows) + CF::ROWS);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + CF::RED);
    uint64_t* empty = full + CF::STAGES;
    uint64_t* bprep = empty + CF::STAGES;
    uint64_t* bsdone = bprep + 1;
    // Per-tile barriers are kept per slot (tile t uses slot t % 2, phase t / 2),
    // so that no waiter is ever two phases behind its barrier (parity waits
    // would alias): P ready, P~ written (P read), O ready, O read. Gathered
    // query tiles, per query slot (tile t uses t % QS, phase t / QS): rows
    // landed with their row table, queries transformed, slot read out.
    uint64_t* bpfull = bsdone + 1;     // [2]
    uint64_t* bptready = bpfull + 2;   // [2]
    uint64_t* bofull = bptready + 2;   // [2]
    uint64_t* bofree = bofull + 2;     // [2]
    uint64_t* qfull = bofree + 2;      // [QS]
    uint64_t* bqready = qfull + CF::QS;  // [QS]
    uint64_t* qfree = bqready + CF::QS;  // [QS]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfree + CF::QS);

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
        }
        for (int j = 0; j < CF::QS; ++j) {
            mbar_init(qfull + j, 1);
            mbar_init(bqready + j, 128);
            mbar_init(qfree + j, 128);
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
                    const int slot = tq % CF::QS, use = tq / CF::QS;
                    int tok[R], lim[R];
#pragma unroll
                    for (int e = 0; e < R; ++e) {
                        const int idx = qbase + t * C + R * lane + e;
                        tok[e] = idx < qend ? perm[(size_t)b * N + idx] : -1;
                        lim[e] = idx < qend ? msort[(size_t)b * N + idx] - c * C : -1;
                    }
                    // the slot's previous tile has been read out (and its row table with it)
                    if (use > 0) ok = __all_sync(0xffffffffu, mbar_wait(qfree + slot, (use - 1) & 1, err));
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
            for (int t2 = max(0, tq - CF::QS); t2 < tq; ++t2)
                mbar_wait(qfull + t2 % CF::QS, (t2 / CF::QS) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id1 = idesc_bf16(C, C, false, false);   // P = Q K^T
            constexpr uint32_t id3 = idesc_bf16(C, D, false, true);    // O = Q S
            constexpr uint32_t idz = idesc_bf16(C, 16, false, false);  // Oz = Q [z]
            constexpr uint32_t id2 = idesc_bf16(C, D, false, true);    // O += P~ V
            constexpr uint32_t id4 = idesc_bf16(D, D, true, true);     // S += K^T V
            const uint32_t pta = smem_u32(pt);
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
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + CF::COL_S, sdesc(kt + kk * 2048, C * 128, 1024),
                             sdesc(vt + kk * 2048, C * 128, 1024), id4, 1u);
                mma_commit(bsdone);
                const uint32_t b3a = smem_u32(b3 + (ci & 1) * CF::B3);
                const uint32_t bza = smem_u32(bz + (ci & 1) * CF::BZ);
                const int ntq = q_tiles(c_begin + ci);
                for (int t = 0; t < ntq && ok; ++t, ++tq) {
                    const int j = tq & 1, k = tq >> 1;  // slot, use of the slot
                    const int qs = tq % CF::QS;  // query slot (gathered tiles)
                    const uint32_t qt = GATHER ? smem_u32(qg + qs * CF::TILE) : st;
                    if (GATHER) ok = mbar_wait(bqready + qs, (tq / CF::QS) & 1, err);
                    if (ok && k > 0) ok = mbar_wait(bptready + j, (k - 1) & 1, err);  // P[j] read two tiles ago
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t ko = (kk / 4) * (C * 128) + (kk % 4) * 32;
                        mma_bf16(tmem + CF::COL_P + CF::p_slot(j), sdesc(qt + ko, 16, 1024), sdesc(kt + ko, 16, 1024),
                                 id1, kk > 0);
                    }
                    mma_commit(bpfull + j);
                    if (k > 0) ok = mbar_wait(bofree + j, (k - 1) & 1, err);  // O[j] read two tiles ago
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = sdesc(qt + (kk / 4) * (C * 128) + (kk % 4) * 32, 16, 1024);
                        mma_bf16(tmem + CF::COL_O + CF::o_slot(j), a, sdesc(b3a + kk * 2048, D * 128, 1024), id3,
                                 kk > 0);
                        if (normalize)
                            mma_bf16(tmem + CF::COL_OZ + CF::oz_slot(j), a,
                                     sdesc(bza + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), idz, kk > 0);
                    }
                    ok = mbar_wait(bptready + j, k & 1, err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t ptj = pta + j * CF::PT;
#pragma unroll
                    for (int kk = 0; kk < C / 16; ++kk)
                        mma_bf16(tmem + CF::COL_O + CF::o_slot(j), sdesc(ptj + (kk / 4) * (C * 128) + (kk % 4) * 32, 16, 1024),
                                 sdesc(vt + kk * 2048, C * 128, 1024), id2, 1u);
                    mma_commit(bofull + j);
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
        // z_prev entry d_k = et (threads et < D), seeded from the prefix
        float zp = (normalize && et < D) ? pre[(size_t)D * D + et] : 0.f;
        // column group (of 8) of the K tiles this thread transforms: the
        // 128-byte swizzle maps 16-byte chunk (et & 7) of its rows (all with
        // the same row & 7) to logical columns 8 * g .. 8 * g + 7
        const int zg = (et & 7) ^ ((et >> 3) & 7);
        {
            // z operand rows 2..15 stay zero (both buffers; rows of 128 bytes)
            for (int c = et; c < 2 * 14 * 8; c += 128)
                reinterpret_cast<uint4*>(bz + (c / 112) * CF::BZ + 2 * 128)[c % 112] = make_uint4(0, 0, 0, 0);
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
            tmem_st_wait();
        }
        // No early exit in this warpgroup: after a failed wait the loops run on
        // without waiting (see cta_abort), so the named barriers stay matched.
        int tq = 0;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
            uint8_t* st = stages + s * CF::STAGE;
            uint4* kt = reinterpret_cast<uint4*>(st + (GATHER ? 0 : CF::TILE));
            mbar_wait(full + s, u & 1, err);
            float cs[8];  // column sums of phi(K) over this thread's rows, group zg
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[e] = 0.f;
            // in groups of 4 chunks, all loads of a group first: a load placed
            // after a shared store could not be moved ahead of it (aliasing)
#pragma unroll
            for (int i0 = 0; i0 < CF::NB * C / 16; i0 += 4) {
                uint4* qt = reinterpret_cast<uint4*>(st);
                uint4 kx[4], qx[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int p = et + 128 * (i0 + i);
                    kx[i] = kt[p];
                    if (!GATHER && mapped) qx[i] = qt[p];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int p = et + 128 * (i0 + i);
                    const int r = (p % (C * 8)) >> 3;
                    const uint4 kn = r < kvalid ? (mapped ? phi8<PHI>(kx[i]) : kx[i]) : make_uint4(0, 0, 0, 0);
                    kt[p] = kn;
                    if (!GATHER && mapped) qt[p] = phi8<PHI>(qx[i]);
                    if (normalize) {
                        float f[8];
                        unpack8(kn, f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) cs[e] += f[e];
                    }
                }
            }
            if (normalize) {
                // lanes l, l ^ 9, l ^ 18, l ^ 27 hold the same column group;
                // lanes 0..7 then publish the warp's sums of all eight groups
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 9);
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 18);
                }
                if (lane < 8) {
                    float4* dst = reinterpret_cast<float4*>(red + (ci & 1) * 4 * D + (warp - 2) * D + zg * 8);
                    dst[0] = make_float4(cs[0], cs[1], cs[2], cs[3]);
                    dst[1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
                }
                named_bar(2, 128);
            }
            if (ci > 0) {
                mbar_wait(bsdone, (ci - 1) & 1, err);
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
            // z_prev -> rows 0 (hi) and 1 (lo) of the z operand (column d_k);
            // then z += the chunk's column sums
            if (normalize && et < D) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(zp);
                const __nv_bfloat16 lo = __float2bfloat16_rn(zp - __bfloat162float(hi));
                uint8_t* zb = bz + (ci & 1) * CF::BZ;
                *reinterpret_cast<__nv_bfloat16*>(zb + sw128_off(0, et)) = hi;
                *reinterpret_cast<__nv_bfloat16*>(zb + sw128_off(1, et)) = lo;
                const float* rp = red + (ci & 1) * 4 * D;
                zp += (rp[et] + rp[D + et]) + (rp[2 * D + et] + rp[3 * D + et]);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);

            if (GATHER) {
                // the gathered query rows of the chunk's tiles: phi in place
                const int ntq = q_tiles(c);
                for (int t = 0; t < ntq; ++t, ++tq) {
                    const int slot = tq % CF::QS;
                    mbar_wait(qfull + slot, (tq / CF::QS) & 1, err);
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
        // M = C accumulators: C = 128 -> lane = row; C = 64 -> rows in lanes
        // 0..15, the two halves of the warp take the two column halves.
        const int i = C == 128 ? sp * 32 + lane : sp * 16 + (lane & 15);
        const int half = (C == 64 && lane >= 16) ? 1 : 0;
        // No early exit in this warpgroup either (named barrier 3 in the
        // causal epilogue); a failed wait only suppresses the output stores.
        bool ok = true;
        int tq = 0;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int kvalid = c < nchunks ? min(C, N - c * C) : 0;
            const int ntq = q_tiles(c);
            for (int t = 0; t < ntq; ++t, ++tq) {
                const int slot = tq & 1, use = tq >> 1;
                const uint32_t lane_s = C == 64 ? lane_base + CF::p_slot(slot) : lane_base;
                uint8_t* pts = pt + slot * CF::PT;
                ok = mbar_wait(bpfull + slot, use & 1, err) && ok;
                // the row table of a gathered tile (written by the TMA warp)
                const int qs = tq % CF::QS;
                if (GATHER) ok = mbar_wait(qfull + qs, (tq / CF::QS) & 1, err) && ok;
                tc_fence_after();
                const int* srow = rows + qs * 2 * C;
                const int lim = GATHER ? srow[C + i] : i;
                const int tok = GATHER ? srow[i] : (i < kvalid ? c * C + i : -1);
                float rs = 0.f;
                if (C == 128) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t r[64];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tmem_ld16(tmem + CF::COL_P + CF::p_slot(slot) + lane_base + 64 * h + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * j));
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
                            *reinterpret_cast<uint4*>(pts + h * (C * 128) + sw128_off(i, 8 * g)) = pack8(f);
                        }
                    }
                } else {
                    uint32_t r[32];
                    tmem_ld16x2<32>(tmem + CF::COL_P + lane_s, *reinterpret_cast<uint32_t(*)[16]>(r));
                    tmem_ld16x2<32>(tmem + CF::COL_P + lane_s + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
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
                        *reinterpret_cast<uint4*>(pts + sw128_off(i, 32 * half + 8 * g)) = pack8(f);
                    }
                    rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                }
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(bptready + slot);
                // epilogue: this thread's segment of output row i
                ok = ok && mbar_wait(bofull + slot, use & 1, err);
                tc_fence_after();
                constexpr int SEG = C == 128 ? D : D / 2;
                uint32_t o[SEG];
#pragma unroll
                for (int j = 0; j < SEG / 16; ++j) {
                    if (C == 128)
                        tmem_ld16(tmem + CF::COL_O + CF::o_slot(slot) + lane_base + 16 * j,
                                  *reinterpret_cast<uint32_t(*)[16]>(o + 16 * j));
                    else
                        tmem_ld16x2<D / 2>(tmem + CF::COL_O + lane_s + 16 * j,
                                           *reinterpret_cast<uint32_t(*)[16]>(o + 16 * j));
                }
                // Oz: a 32x32b load must start at the warp's sub-partition
                // base; with 64-row chunks slot 1 sits in lanes 16..31 and is
                // picked out below with a shuffle
                uint32_t oz[2];
                tmem_ld2(tmem + CF::COL_OZ + lane_base + (C == 64 ? 0u : CF::oz_slot(slot)), oz);
                tmem_ld_wait();
                tc_fence_before();
                // gathered rows: this thread's copy-out rows, read before the
                // slot (and its row table) is handed back
                constexpr int NC = C * D / 8 / 128;
                int dst_row[GATHER ? NC : 1];
                if (GATHER) {
#pragma unroll
                    for (int j = 0; j < NC; ++j) dst_row[j] = srow[(threadIdx.x - 192 + 128 * j) / (D / 8)];
                }
                mbar_arrive(bofree + slot);
                if (GATHER) mbar_arrive(qfree + qs);  // the query slot and its row table are read
                float den = rs + __uint_as_float(oz[0]) + __uint_as_float(oz[1]);
                if (C == 64) den = __shfl_sync(0xffffffffu, den, (lane & 15) + 16 * slot);
                const float inv = normalize ? __frcp_rn(den) : 1.0f;
                if (!GATHER) {
                    // causal: the chunk's rows are contiguous; stage them and
                    // write the tile with one TMA store (rows past N are clipped)
                    const int et2 = threadIdx.x - 192;
                    if (et2 == 0) bulk_wait_read0();
                    named_bar(3, 128);
#pragma unroll
                    for (int g = 0; g < SEG / 8; ++g) {
                        const int col = half * SEG + 8 * g;
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[8 * g + e]) * inv;
                        *reinterpret_cast<uint4*>(stg + (col / 64) * (C * 128) + sw128_off(i, col % 64)) = pack8(f);
                    }
                    fence_async_smem();
                    named_bar(3, 128);
                    if (et2 == 0 && ok) {
#pragma unroll
                        for (int bx = 0; bx < CF::NB; ++bx)
                            tma_store_3d(&mOut, stg + bx * (C * 128), bx * 64, c * C, bh);
                        bulk_commit();
                    }
                } else {
                    // gathered rows: stage the tile, then copy it out a full row
                    // per 8 (d = 64) or 16 (d = 128) consecutive threads
                    const int et2 = threadIdx.x - 192;
                    named_bar(3, 128);  // the previous tile's copy-out has read the staging tile
#pragma unroll
                    for (int g = 0; g < SEG / 8; ++g) {
                        const int col = half * SEG + 8 * g;
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[8 * g + e]) * inv;
                        *reinterpret_cast<uint4*>(stg + (col / 64) * (C * 128) + sw128_off(i, col % 64)) = pack8(f);
                    }
                    named_bar(3, 128);
#pragma unroll
                    for (int j = 0; j < NC; ++j) {
                        const int p = et2 + 128 * j;
                        const int r = p / (D / 8), col = (p % (D / 8)) * 8;
                        if (ok && dst_row[j] >= 0)
                            *reinterpret_cast<uint4*>(out + hoff + (size_t)dst_row[j] * D + col) =
                                *reinterpret_cast<const uint4*>(stg + (col / 64) * (C * 128) + sw128_off(r, col % 64));
                    }
                    (void)tok;
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

template <int D, int C, bool GATHER, int PHI>
cudaError_t launch_chunked(const Problem& p, const void* q, const void* k, const void* v,
                           const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                           const int32_t* bins, const int32_t* msort, int nbins, void* out, uint32_t* err,
                           cudaStream_t st) {
    if (block_tokens % C != 0) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv, mo;
    // gathered queries: a 2-D row map for tile::gather4
    cudaError_t e = GATHER ? make_row_map(&mq, q, D, p.bh() * p.N) : make_map(&mq, q, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mk, k, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mo, out, D, p.N, p.bh(), C);
    if (e != cudaSuccess) return e;
    using CF = SwCfg<D, C, GATHER>;
    constexpr size_t smem = CF::SMEM;
    e = ensure_smem<tc_sweep_kernel<D, C, GATHER, PHI>>(smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nblk, (unsigned)p.bh());
    return launch_pdl(tc_sweep_kernel<D, C, GATHER, PHI>, grid, dim3(CF::THREADS), smem, st, mq, mk, mv, mo,
                      prefix, p.H, p.N, block_tokens, nblk, perm, bins, msort, nbins, p.normalize,
                      static_cast<__nv_bfloat16*>(out), err);
}

// one kernel per feature map (see phi8)
template <int D, int C, bool GATHER>
cudaError_t launch_phi(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                       int block_tokens, int nblk, const int32_t* perm, const int32_t* bins, const int32_t* msort,
                       int nbins, void* out, uint32_t* err, cudaStream_t st) {
    switch (p.phi) {
        case PHI_RELU1:
            return launch_chunked<D, C, GATHER, PHI_RELU1>(p, q, k, v, prefix, block_tokens, nblk, perm, bins,
                                                           msort, nbins, out, err, st);
        case PHI_ELU1:
            return launch_chunked<D, C, GATHER, PHI_ELU1>(p, q, k, v, prefix, block_tokens, nblk, perm, bins,
                                                          msort, nbins, out, err, st);
        default:
            return launch_chunked<D, C, GATHER, PHI_IDENTITY>(p, q, k, v, prefix, block_tokens, nblk, perm, bins,
                                                              msort, nbins, out, err, st);
    }
}

}  // namespace

cudaError_t tc_chunked(const Problem& p, int chunk, const void* q, const void* k, const void* v,
                       const float* prefix, int block_tokens, int nblk, const int32_t* perm,
                       const int32_t* bins, const int32_t* msort, int nbins, void* out, uint32_t* err,
                       cudaStream_t st) {
    const int C = tc_chunk(p, chunk);
    const bool g = perm != nullptr;
#define LA_CH(D_, C_, G_) \
    return launch_phi<D_, C_, G_>(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins, out, err, st)
    if (p.d == 128) return tc_chunked_t(p, q, k, v, prefix, block_tokens, nblk, perm, bins, msort, nbins, out, err, st);
    if (C == 64) {
        if (g) LA_CH(64, 64, true);
        LA_CH(64, 64, false);
    }
    if (g) LA_CH(64, 128, true);
    LA_CH(64, 128, false);
#undef LA_CH
}

}  // namespace la
