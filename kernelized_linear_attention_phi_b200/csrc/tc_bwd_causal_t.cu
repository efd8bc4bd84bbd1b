// Gradients of the causal form at d = 128 on tcgen05 tensor cores (bf16,
// 64-token chunks): the same two sweeps as the d = 64 kernels
// (tc_bwd_causal.cu), laid out for d = 128.
//
// First sweep, one CTA per (block, head), chunks in order (A = phi(Q),
// B = phi(K), V, g the chunk's rows; S, z the running state seeded from the
// block's prefix record):
//   S_prev, z_prev -> bf16 operands                           [prep]
//   S += B^T V, z += B^T 1                                     [MMA, M = d_k]
//   P = A B^T -> P~ (j <= i, bf16), rowsum                     [MMA, mask]
//   O = A S_prev + P~ V, den = rowsum + A [z_hi; z_lo]         [MMA]
//   gn = g / den (over the dO tile, then stored), gden = -(g . out) / den
//   dA = GN S_prev^T ; W = GN V^T -> W~ = (W + gden 1^T) masked
//   G += A^T GN, h += A^T [gden_hi; gden_lo]                    [MMA, M = d_k]
//   dA += W~ B ; dq = phi'(q) (dA + gden z_prev)               [MMA, epilogue]
// Second sweep, chunks from the last to the first, with the running suffix
// G, h of the queries after the chunk, seeded from the block's suffix record:
//   G_next, h_next -> bf16 operand, fp32 copy                  [prep]
//   G += A^T GN, h += A^T [gden_hi; gden_lo]                   [MMA]
//   P^T = B A^T -> P~^T (i >= j, bf16)                         [MMA, mask]
//   dV = B G_next + P~^T GN ; dB = V G_next^T                  [MMA]
//   W^T = V GN^T -> W~^T = (W^T + 1 gden^T) masked             [MMA, mask]
//   dB += W~^T A ; dk = phi'(k) (dB + h_next), dv = dV         [MMA, epilogue]
//
// At d = 128 the running states (S and G, M = d_k = 128) take 128 TMEM
// columns each, with every lane a row, and z, h 16 columns each; the
// per-chunk M = 64 accumulators pair up in the two 16-lane halves of each
// sub-partition as at d = 64 (O / dA, dV / dB: 128 columns), P and W share
// 64 columns. One CTA per SM: two stages of Q, K, V and dO (or GN) tiles of
// [64 x 128] (two 64-column swizzle boxes each) and the bf16 copy of the
// state ([128 x 128], two atoms along d_v, double-buffered) take most of the
// shared memory. Warp roles as at d = 64: warp 0 TMA, warp 1 TMEM owner and
// MMA issuer, warps 2-5 prep, warps 6-9 masks and epilogues (row
// 16 sp + (lane & 15) of the chunk; the warp halves take the two 64-column
// halves of d, or the two 32-column halves of the chunk).

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kD = 128, kC = 64;
constexpr int kBox = kC * 128;        // one [64 x 64] bf16 box of a tile (8 KB)
constexpr int kTile = 2 * kBox;       // one [64 x 128] bf16 tile
constexpr int kAtom = kD * 128;       // one [128 x 64] bf16 atom of the state copy (16 KB)
constexpr uint32_t kLane16 = 16u << 16;

// Loads one [64 x 128] tile as its two boxes.
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row, int bh) {
    tma_load_3d(dst, map, bar, 0, row, bh);
    tma_load_3d(dst + kBox, map, bar, 64, row, bh);
}
__device__ __forceinline__ void store_tile(const CUtensorMap* map, const uint8_t* src, int row, int bh) {
    tma_store_3d(map, src, 0, row, bh);
    tma_store_3d(map, src + kBox, 64, row, bh);
}
// Byte offset of the 8 columns at `col` (a multiple of 8) of `row` in a
// [64 x 128] tile.
__device__ __forceinline__ uint32_t tile_off(int row, int col) { return (col / 64) * kBox + sw128_off(row, col % 64); }

// phi in place over one [64 x 128] tile (keys past `valid` zeroed when `zero`),
// relu'(x) bits per 8-column group into sg[row * 16 + group] when `bits`.
// Thread et of 128 takes 16-byte chunks et + 128 j.
template <int PHI, bool MAPPED>
__device__ __forceinline__ void transform_tile(uint8_t* tb, int et, int valid, bool zero, uint8_t* sg, bool bits) {
    uint4* t = reinterpret_cast<uint4*>(tb);
    uint4 x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = t[et + 128 * j];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int p = et + 128 * j, box = p >> 9, r = (p & 511) >> 3;
        if (PHI == PHI_RELU1 && bits) sg[r * 16 + box * 8 + ((p & 7) ^ (r & 7))] = static_cast<uint8_t>(positive_bits(x[j]));
        uint4 y = MAPPED ? phi8<PHI>(x[j]) : x[j];
        if (zero && r >= valid) y = make_uint4(0, 0, 0, 0);
        if (MAPPED || zero) t[p] = y;
    }
}

// Row a of an fp32 [128 x 128] M = 128 accumulator at TMEM column `col`
// (lane a of the warp's sub-partition) into row a of a bf16 [d_k][d_v]
// state copy (two atoms along d_v).
__device__ __forceinline__ void state_row_to_bf16(uint32_t taddr, uint8_t* dst, int a) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t r[64];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld16(taddr + 64 * h + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * j));
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * g + e]);
            *reinterpret_cast<uint4*>(dst + h * kAtom + sw128_off(a, 8 * g)) = pack8(f);
        }
    }
}

// Seeds row a (lane a of the warp's sub-partition) of an M = 128 state at
// TMEM column `col` from rec[a][0..127], and the 16 columns at `zcol` with
// rec[128 * 128 + a] (or 0): every column (z, whose MMA against the all-ones
// operand adds the same sum to each) or column 0 alone (h, whose MMA adds
// A^T gden_hi to column 0 and A^T gden_lo to column 1).
__device__ __forceinline__ void seed_state_row(uint32_t tcol, uint32_t tzcol, const float* rec, int a, bool with_z,
                                               bool every_col) {
#pragma unroll
    for (int c0 = 0; c0 < kD; c0 += 16) {
        uint32_t r[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const float4 x = reinterpret_cast<const float4*>(rec + (size_t)a * kD + c0)[q4];
            r[4 * q4] = __float_as_uint(x.x);
            r[4 * q4 + 1] = __float_as_uint(x.y);
            r[4 * q4 + 2] = __float_as_uint(x.z);
            r[4 * q4 + 3] = __float_as_uint(x.w);
        }
        tmem_st16(tcol + c0, r);
    }
    uint32_t r[16];
    const uint32_t zv = with_z ? __float_as_uint(rec[(size_t)kD * kD + a]) : 0u;
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = (every_col || e == 0) ? zv : 0u;
    tmem_st16(tzcol, r);
    tmem_st_wait();
}

// 64 columns (this warp half's) of row i of an M = 64 accumulator whose rows
// sit in lanes 0..15 of each sub-partition from `taddr` (the lane base of the
// warp, plus 16 lanes for the second accumulator of a pair).
__device__ __forceinline__ void ld_half64(uint32_t taddr, uint32_t (&r)[64]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_ld16x2<64>(taddr + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(r + 16 * j));
    tmem_ld_wait();
}
// 32 columns of the chunk (this warp half's) of row i of a [64 x 64] M = 64 accumulator.
__device__ __forceinline__ void ld_half32(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_ld16x2<32>(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
    tmem_ld16x2<32>(taddr + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
    tmem_ld_wait();
}

// ---------------------------------------------------------------------------
// First sweep: dq, gn, gden and the blocks' (G, h)
// ---------------------------------------------------------------------------
struct QtCfg {
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 4 * kTile;   // Q, K, V, dO (g, then gn, then dq)
    static constexpr int B3 = 2 * kAtom;      // S_prev bf16 [d_k][d_v] (x2)
    static constexpr int BZ = 2 * 16 * 128;   // [z_hi; z_lo; 0], K-major over d_k: two boxes (x2)
    static constexpr int ONES = 16 * kC * 2;  // all-ones [16][64], K-major
    static constexpr int PT = kC * kC * 2;    // P~, then W~ [query][key], K-major
    static constexpr int BGD = 16 * kC * 2;   // [gden_hi; gden_lo; 0] over the chunk, K-major
    static constexpr int SGN = kC * kD / 8;   // relu'(q) bits (x STAGES)
    static constexpr int ZF = 2 * kD * 4;     // z_prev fp32 (x2)
    // TMEM columns
    static constexpr int COL_S = 0;     // S, M = 128 (row d_k in lane d_k)
    static constexpr int COL_G = 128;   // G, M = 128
    static constexpr int COL_Z = 256;   // z, M = 128 (16 equal columns)
    static constexpr int COL_H = 272;   // h, M = 128
    static constexpr int COL_P = 288;   // P, then W (M = 64)
    static constexpr int COL_O = 352;   // O (lanes 0-15), dA (lanes 16-31), M = 64, 128 columns
    static constexpr int COL_OZ = 480;  // den terms (M = 64)
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NBAR = 2 * STAGES + 11;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * B3 + 2 * BZ + ONES + PT + BGD + STAGES * SGN +
                                   ZF + 8 * NBAR + 16;
    static constexpr int THREADS = 320;
    static_assert(COL_OZ + 16 <= (int)TMEM_COLS, "TMEM");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && B3 % 1024 == 0 && BZ % 1024 == 0, "1024-byte aligned operand tiles");
};

template <int PHI>
__global__ void __launch_bounds__(QtCfg::THREADS, 1)
tc_bwd_causal_q_t_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                         const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mGo,
                         const __grid_constant__ CUtensorMap mGn, const __grid_constant__ CUtensorMap mDq,
                         const float* __restrict__ prefix, int N, int block_tokens, int nblk, int normalize,
                         float* __restrict__ gden_out, float* __restrict__ grec, uint32_t* __restrict__ err) {
    using CF = QtCfg;
    constexpr int D = kD, C = kC;
    constexpr bool mapped = PHI != PHI_IDENTITY;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* b3 = stages + CF::STAGES * CF::STAGE;
    uint8_t* bz = b3 + 2 * CF::B3;
    uint8_t* ones = bz + 2 * CF::BZ;
    uint8_t* pt = ones + CF::ONES;
    uint8_t* bgd = pt + CF::PT;
    uint8_t* sgn = bgd + CF::BGD;
    float* zf = reinterpret_cast<float*>(sgn + CF::STAGES * CF::SGN);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(zf) + CF::ZF);
    uint64_t* empty = full + CF::STAGES;  // MMA done with the stage and dq stored from it
    uint64_t* bprep = empty + CF::STAGES; // phi(Q), phi(K) and the S_prev, z_prev operands ready
    uint64_t* bsdone = bprep + 1;         // S, z updated with the chunk
    uint64_t* pfull = bsdone + 1;         // P ready
    uint64_t* ptready = pfull + 1;        // P~ written (P read)
    uint64_t* ofull = ptready + 1;        // O, den terms ready
    uint64_t* gnready = ofull + 1;        // gn, gden operands written (O read)
    uint64_t* wfull = gnready + 1;        // W ready (and G, h terms issued)
    uint64_t* wtready = wfull + 1;        // W~ written (W read)
    uint64_t* dafull = wtready + 1;       // dA ready
    uint64_t* dafree = dafull + 1;        // dA read
    uint64_t* gfull = dafree + 1;         // the block's G, h complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gfull + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y;
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    const int nci = min(nchunks, c_begin + block_tokens / C) - c_begin;

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 2);
        }
        mbar_init(bprep, 128);
        mbar_init(bsdone, 1);
        mbar_init(pfull, 1);
        mbar_init(ptready, 128);
        mbar_init(ofull, 1);
        mbar_init(gnready, 128);
        mbar_init(wfull, 1);
        mbar_init(wtready, 128);
        mbar_init(dafull, 1);
        mbar_init(dafree, 128);
        mbar_init(gfull, 1);
        fence_mbar_init();
        tma_prefetch_map(&mQ);
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
        tma_prefetch_map(&mGo);
        tma_prefetch_map(&mGn);
        tma_prefetch_map(&mDq);
    }
    if (warp == 1) tmem_alloc(tmem_slot, CF::TMEM_COLS);
    {
        // all-ones operand; z and gden operands zero (their rows 0 and 1 are rewritten)
        const uint4 one8 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (int c = threadIdx.x; c < CF::ONES / 16; c += CF::THREADS) reinterpret_cast<uint4*>(ones)[c] = one8;
        for (int c = threadIdx.x; c < 2 * CF::BZ / 16; c += CF::THREADS) reinterpret_cast<uint4*>(bz)[c] = make_uint4(0, 0, 0, 0);
        for (int c = threadIdx.x; c < CF::BGD / 16; c += CF::THREADS) reinterpret_cast<uint4*>(bgd)[c] = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The TMA producer loads only the caller's Q, K, V, dO; every other warp
    // waits for the previous kernel (the block-state scan) first.
    if (warp != 0) pdl_wait();

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
                load_tile(st, &mQ, full + s, row, bh);
                load_tile(st + kTile, &mK, full + s, row, bh);
                load_tile(st + 2 * kTile, &mV, full + s, row, bh);
                load_tile(st + 3 * kTile, &mGo, full + s, row, bh);
                issued[s] = u + 1;
            }
            for (int s = 0; s < CF::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id_s = idesc_bf16(D, D, true, true);      // S += B^T V, G += A^T GN
            constexpr uint32_t id_z = idesc_bf16(D, 16, true, false);    // z += B^T 1, h += A^T [gden]
            constexpr uint32_t id_p = idesc_bf16(C, C, false, false);    // P = A B^T, W = GN V^T
            constexpr uint32_t id_o = idesc_bf16(C, D, false, true);     // O = A S_prev, O += P~ V, dA += W~ B
            constexpr uint32_t id_oz = idesc_bf16(C, 16, false, false);  // den = A [z]
            constexpr uint32_t id_a = idesc_bf16(C, D, false, false);    // dA = GN S_prev^T
            const uint32_t pta = smem_u32(pt), onesa = smem_u32(ones), gda = smem_u32(bgd);
            // K-major operand over d (two boxes): step kk of 16 columns
            auto kmaj = [](uint32_t t, int kk) { return sdesc(t + (kk / 4) * kBox + (kk % 4) * 32, 16, 1024); };
            // a tile as an MN-major operand over d (M or N = 128: two boxes), step kk of 16 rows
            auto mnmaj = [](uint32_t t, int kk) { return sdesc(t + kk * 2048, kBox, 1024); };
            bool ok = true;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t qt = smem_u32(stages + s * CF::STAGE), kt = qt + kTile, vt = kt + kTile,
                               gt = vt + kTile;
                const uint32_t b3a = smem_u32(b3 + (ci & 1) * CF::B3), bza = smem_u32(bz + (ci & 1) * CF::BZ);
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t a = mnmaj(kt, kk);  // B^T, MN-major
                    mma_bf16(tmem + CF::COL_S, a, mnmaj(vt, kk), id_s, 1u);
                    if (normalize) mma_bf16(tmem + CF::COL_Z, a, sdesc(onesa + kk * 32, 16, 1024), id_z, 1u);
                }
                mma_commit(bsdone);
                if (ci > 0) {
                    ok = mbar_wait(wtready, (ci - 1) & 1, err);  // W of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(tmem + CF::COL_P, kmaj(qt, kk), kmaj(kt, kk), id_p, kk > 0 ? 1u : 0u);
                mma_commit(pfull);
                if (ci > 0) {
                    ok = mbar_wait(gnready, (ci - 1) & 1, err);  // O of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = kmaj(qt, kk);
                    mma_bf16(tmem + CF::COL_O, a, sdesc(b3a + kk * 2048, kAtom, 1024), id_o, kk > 0 ? 1u : 0u);
                    if (normalize)
                        mma_bf16(tmem + CF::COL_OZ, a, sdesc(bza + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_oz,
                                 kk > 0 ? 1u : 0u);
                }
                ok = mbar_wait(ptready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + CF::COL_O, sdesc(pta + kk * 32, 16, 1024), mnmaj(vt, kk), id_o, 1u);
                mma_commit(ofull);
                ok = mbar_wait(gnready, ci & 1, err);
                if (ok && ci > 0) ok = mbar_wait(dafree, (ci - 1) & 1, err);  // dA of the last chunk read
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // dA = GN S_prev^T (S_prev read K-major over d_v)
                    mma_bf16(tmem + CF::COL_O + kLane16, kmaj(gt, kk),
                             sdesc(b3a + (kk / 4) * kAtom + (kk % 4) * 32, 16, 1024), id_a, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // W = GN V^T
                    mma_bf16(tmem + CF::COL_P, kmaj(gt, kk), kmaj(vt, kk), id_p, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {  // G += A^T GN, h += A^T [gden]
                    const uint64_t a = mnmaj(qt, kk);
                    const uint32_t accum = (ci == 0 && kk == 0) ? 0u : 1u;
                    mma_bf16(tmem + CF::COL_G, a, mnmaj(gt, kk), id_s, accum);
                    if (normalize) mma_bf16(tmem + CF::COL_H, a, sdesc(gda + kk * 32, 16, 1024), id_z, accum);
                }
                mma_commit(wfull);
                ok = mbar_wait(wtready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dA += W~ B
                    mma_bf16(tmem + CF::COL_O + kLane16, sdesc(pta + kk * 32, 16, 1024), mnmaj(kt, kk), id_o, 1u);
                mma_commit(dafull);
                mma_commit(empty + s);
                if (ci == nci - 1) mma_commit(gfull);
            }
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int a = sp * 32 + lane;  // the state row (d_k) this thread owns in TMEM
        // seed S, z with the block's prefix
        seed_state_row(tmem + CF::COL_S + lane_base, tmem + CF::COL_Z + lane_base,
                       prefix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D), a, normalize != 0, true);
        // No early exit in this warpgroup: after a failed wait the loop runs
        // on without waiting (see cta_abort).
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int kvalid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            mbar_wait(full + s, u & 1, err);
            uint8_t* sg = sgn + s * CF::SGN;
            transform_tile<PHI, mapped>(st + kTile, et, kvalid, true, sg, false);  // keys past N stay zero
            transform_tile<PHI, mapped>(st, et, C, false, sg, mapped);
            if (ci > 0) {
                mbar_wait(bsdone, (ci - 1) & 1, err);
                tc_fence_after();
            }
            // S_prev -> bf16 [d_k][d_v]; z_prev -> rows 0 (hi), 1 (lo) of the z operand and fp32
            uint8_t* b3b = b3 + (ci & 1) * CF::B3;
            state_row_to_bf16(tmem + CF::COL_S + lane_base, b3b, a);
            float zv = 0.f;
            if (normalize) {
                uint32_t r[16];
                tmem_ld16(tmem + CF::COL_Z + lane_base, r);
                tmem_ld_wait();
                zv = __uint_as_float(r[0]);
                const __nv_bfloat16 zh = __float2bfloat16_rn(zv);
                const __nv_bfloat16 zl = __float2bfloat16_rn(zv - __bfloat162float(zh));
                uint8_t* base = bz + (ci & 1) * CF::BZ + (a / 64) * 2048;
                *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(0, a % 64)) = zh;
                *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(1, a % 64)) = zl;
            }
            zf[(ci & 1) * D + a] = zv;
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);
        }
    } else {
        // ---------------- mask and epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int i = sp * 16 + (lane & 15);  // query row of the chunk
        const int half = lane >> 4;           // this thread's half of the columns
        const int et2 = threadIdx.x - 192;
        // No early exit in this warpgroup (named barrier 3); a failed wait
        // only suppresses the stores.
        bool ok = true;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES;
            const int valid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            uint8_t* gt = st + 3 * kTile;  // dO: g, then gn, then dq
            // ---- P~ = P masked (key j <= query i), row sums
            ok = mbar_wait(pfull, ci & 1, err) && ok;
            tc_fence_after();
            float rs = 0.f;
            {
                uint32_t r[32];
                ld_half32(tmem + CF::COL_P + lane_base, r);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * half + 8 * g + e;
                        f[e] = j <= i ? __uint_as_float(r[8 * g + e]) : 0.f;
                        rs += f[e];
                    }
                    *reinterpret_cast<uint4*>(pt + sw128_off(i, 32 * half + 8 * g)) = pack8(f);
                }
            }
            rs += __shfl_xor_sync(0xffffffffu, rs, 16);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ptready);
            // ---- out, gn (over g in the dO tile), gden
            ok = ok && mbar_wait(ofull, ci & 1, err);
            tc_fence_after();
            uint32_t o[64];
            ld_half64(tmem + CF::COL_O + lane_base, o);
            uint32_t oz[2] = {0u, 0u};
            if (normalize) {
                tmem_ld2(tmem + CF::COL_OZ + lane_base, oz);  // rows in lanes 0..15
                tmem_ld_wait();
            }
            float den = rs + __uint_as_float(oz[0]) + __uint_as_float(oz[1]);
            den = __shfl_sync(0xffffffffu, den, lane & 15);
            const float inv = normalize ? __frcp_rn(den) : 1.0f;
            float dot = 0.f;  // g . O over this half
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                uint4* p = reinterpret_cast<uint4*>(gt + tile_off(i, 64 * half + 8 * g));
                float f[8];
                unpack8(*p, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dot += f[e] * __uint_as_float(o[8 * g + e]);
                    f[e] *= inv;
                }
                *p = pack8(f);
            }
            dot += __shfl_xor_sync(0xffffffffu, dot, 16);
            const float gden = normalize ? -dot * inv * inv : 0.f;
            if (half == 0) {
                if (normalize) {
                    const __nv_bfloat16 gh = __float2bfloat16_rn(gden);
                    const __nv_bfloat16 gl = __float2bfloat16_rn(gden - __bfloat162float(gh));
                    *reinterpret_cast<__nv_bfloat16*>(bgd + sw128_off(0, i)) = gh;
                    *reinterpret_cast<__nv_bfloat16*>(bgd + sw128_off(1, i)) = gl;
                }
                if (i < valid) gden_out[(size_t)bh * N + (size_t)c * C + i] = gden;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(gnready);
            named_bar(3, 128);  // the gn tile is complete: store it for the second sweep
            if (et2 == 0 && ok) {
                store_tile(&mGn, gt, c * C, bh);
                bulk_commit();
            }
            // ---- W~ = (W + gden_i) masked (key j <= query i)
            ok = ok && mbar_wait(wfull, ci & 1, err);
            tc_fence_after();
            {
                uint32_t r[32];
                ld_half32(tmem + CF::COL_P + lane_base, r);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 32 * half + 8 * g + e;
                        f[e] = j <= i ? __uint_as_float(r[8 * g + e]) + gden : 0.f;
                    }
                    *reinterpret_cast<uint4*>(pt + sw128_off(i, 32 * half + 8 * g)) = pack8(f);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(wtready);
            // ---- dq = phi'(q) (dA + gden z_prev) over the dO tile
            ok = ok && mbar_wait(dafull, ci & 1, err);
            tc_fence_after();
            uint32_t da[64];
            ld_half64(tmem + CF::COL_O + lane_base + kLane16, da);
            tc_fence_before();
            mbar_arrive(dafree);
            if (et2 == 0) bulk_wait_read0();  // the gn store has read the tile
            named_bar(3, 128);
            const float* zb = zf + (ci & 1) * D;
            const uint8_t* sg = sgn + s * CF::SGN + i * 16;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const int col = 64 * half + 8 * g;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(da[8 * g + e]) + gden * zb[col + e];
                const uint4 pq = PHI == PHI_ELU1 ? *reinterpret_cast<const uint4*>(st + tile_off(i, col))
                                                 : make_uint4(0, 0, 0, 0);
                times_phi_grad<PHI>(f, PHI == PHI_RELU1 ? sg[col / 8] : 0u, pq);
                *reinterpret_cast<uint4*>(gt + tile_off(i, col)) = pack8(f);
            }
            fence_async_smem();
            named_bar(3, 128);
            if (et2 == 0) {
                if (ok) {
                    store_tile(&mDq, gt, c * C, bh);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(empty + s);
            }
        }
        // ---- the block's (G, h): row d_k = a of the M = 128 accumulators
        ok = ok && mbar_wait(gfull, 0, err);
        tc_fence_after();
        {
            const int a = sp * 32 + lane;
            float* rec = grec + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t v[64];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    tmem_ld16(tmem + CF::COL_G + lane_base + 64 * h + 16 * j, *reinterpret_cast<uint32_t(*)[16]>(v + 16 * j));
                tmem_ld_wait();
                float4* o4 = reinterpret_cast<float4*>(rec + (size_t)a * D + 64 * h);
#pragma unroll
                for (int q4 = 0; q4 < 16; ++q4)
                    o4[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                         __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
            }
            uint32_t hr[2] = {0u, 0u};
            if (normalize) {
                tmem_ld2(tmem + CF::COL_H + lane_base, hr);
                tmem_ld_wait();
            }
            rec[(size_t)D * D + a] = normalize ? __uint_as_float(hr[0]) + __uint_as_float(hr[1]) : 0.f;
        }
        if (et2 == 0) bulk_wait0();  // the stores have landed
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CF::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Second sweep: dk, dv
// ---------------------------------------------------------------------------
struct KtCfg {
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 4 * kTile;   // Q, K, V, GN (K, V then dk, dv)
    static constexpr int BGM = 2 * kAtom;     // G_next bf16 [d_k][d_v] (x2)
    static constexpr int PT = kC * kC * 2;    // P~^T, then W~^T [key][query], K-major
    static constexpr int BGD = 16 * kC * 2;   // [gden_hi; gden_lo; 0] over the chunk (x2)
    static constexpr int SGN = kC * kD / 8;   // relu'(k) bits (x STAGES)
    static constexpr int VEC = (2 * kD + 2 * kC) * 4;  // h_next [2][D] and the chunk's gden [2][C], fp32
    static constexpr int COL_G = 0;    // G, M = 128
    static constexpr int COL_H = 128;  // h, M = 128
    static constexpr int COL_P = 144;  // P^T, then W^T (M = 64)
    static constexpr int COL_D = 208;  // dV (lanes 0-15), dB (lanes 16-31), M = 64, 128 columns
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NBAR = 2 * STAGES + 9;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * BGM + PT + 2 * BGD + STAGES * SGN + VEC +
                                   8 * NBAR + 16;
    static constexpr int THREADS = 320;
    static_assert(COL_D + 128 <= (int)TMEM_COLS, "TMEM");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(STAGE % 1024 == 0 && BGM % 1024 == 0 && PT % 1024 == 0 && BGD % 1024 == 0, "aligned operand tiles");
};

template <int PHI>
__global__ void __launch_bounds__(KtCfg::THREADS, 1)
tc_bwd_causal_kv_t_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                          const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mGn,
                          const __grid_constant__ CUtensorMap mDk, const __grid_constant__ CUtensorMap mDv,
                          const float* __restrict__ suffix, const float* __restrict__ gden_in, int N,
                          int block_tokens, int nblk, int normalize, uint32_t* __restrict__ err) {
    using CF = KtCfg;
    constexpr int D = kD, C = kC;
    constexpr bool mapped = PHI != PHI_IDENTITY;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* gbm = stages + CF::STAGES * CF::STAGE;
    uint8_t* pt = gbm + 2 * CF::BGM;
    uint8_t* bgd = pt + CF::PT;
    uint8_t* sgn = bgd + 2 * CF::BGD;
    float* hf = reinterpret_cast<float*>(sgn + CF::STAGES * CF::SGN);  // [2][D]
    float* gdf = hf + 2 * D;                                           // [2][C]
    uint64_t* full = reinterpret_cast<uint64_t*>(gdf + 2 * C);
    uint64_t* empty = full + CF::STAGES;   // MMA done with the stage and dk, dv stored from it
    uint64_t* bprep = empty + CF::STAGES;  // phi(Q), phi(K), gden and the G_next operand ready
    uint64_t* gdone = bprep + 1;           // G, h updated with the chunk
    uint64_t* pfull = gdone + 1;
    uint64_t* ptready = pfull + 1;
    uint64_t* wfull = ptready + 1;
    uint64_t* wtready = wfull + 1;
    uint64_t* dfull = wtready + 1;         // dV, dB ready
    uint64_t* dfree = dfull + 1;           // dV, dB read
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfree + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int blk = blockIdx.x;
    const int bh = blockIdx.y;
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    const int nci = min(nchunks, c_begin + block_tokens / C) - c_begin;
    auto chunk_of = [&](int ci) { return c_begin + nci - 1 - ci; };  // last to first

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 2);
        }
        mbar_init(bprep, 128);
        mbar_init(gdone, 1);
        mbar_init(pfull, 1);
        mbar_init(ptready, 128);
        mbar_init(wfull, 1);
        mbar_init(wtready, 128);
        mbar_init(dfull, 1);
        mbar_init(dfree, 128);
        fence_mbar_init();
        tma_prefetch_map(&mQ);
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
        tma_prefetch_map(&mGn);
        tma_prefetch_map(&mDk);
        tma_prefetch_map(&mDv);
    }
    if (warp == 1) tmem_alloc(tmem_slot, CF::TMEM_COLS);
    for (int c = threadIdx.x; c < 2 * CF::BGD / 16; c += CF::THREADS) reinterpret_cast<uint4*>(bgd)[c] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // GN comes from an earlier kernel of the call, so the producer waits too
    pdl_wait();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued[CF::STAGES] = {};
            for (int ci = 0; ci < nci; ++ci) {
                const int s = ci % CF::STAGES, u = ci / CF::STAGES;
                if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1, err)) break;
                mbar_arrive_expect_tx(full + s, CF::STAGE);
                uint8_t* st = stages + s * CF::STAGE;
                const int row = chunk_of(ci) * C;
                load_tile(st, &mQ, full + s, row, bh);
                load_tile(st + kTile, &mK, full + s, row, bh);
                load_tile(st + 2 * kTile, &mV, full + s, row, bh);
                load_tile(st + 3 * kTile, &mGn, full + s, row, bh);
                issued[s] = u + 1;
            }
            for (int s = 0; s < CF::STAGES; ++s)
                if (issued[s] > 0) mbar_wait(full + s, (issued[s] - 1) & 1, err, false);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t id_g = idesc_bf16(D, D, true, true);      // G += A^T GN
            constexpr uint32_t id_h = idesc_bf16(D, 16, true, false);    // h += A^T [gden]
            constexpr uint32_t id_p = idesc_bf16(C, C, false, false);    // P^T = B A^T, W^T = V GN^T
            constexpr uint32_t id_n = idesc_bf16(C, D, false, true);     // dV = B G, dV += P~^T GN, dB += W~^T A
            constexpr uint32_t id_t = idesc_bf16(C, D, false, false);    // dB = V G^T
            const uint32_t pta = smem_u32(pt);
            auto kmaj = [](uint32_t t, int kk) { return sdesc(t + (kk / 4) * kBox + (kk % 4) * 32, 16, 1024); };
            auto mnmaj = [](uint32_t t, int kk) { return sdesc(t + kk * 2048, kBox, 1024); };
            bool ok = true;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t qt = smem_u32(stages + s * CF::STAGE), kt = qt + kTile, vt = kt + kTile,
                               nt = vt + kTile;
                const uint32_t gb = smem_u32(gbm + (ci & 1) * CF::BGM), gda = smem_u32(bgd + (ci & 1) * CF::BGD);
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t a = mnmaj(qt, kk);  // A^T, MN-major
                    mma_bf16(tmem + CF::COL_G, a, mnmaj(nt, kk), id_g, 1u);
                    if (normalize) mma_bf16(tmem + CF::COL_H, a, sdesc(gda + kk * 32, 16, 1024), id_h, 1u);
                }
                mma_commit(gdone);
                if (ci > 0) {
                    ok = mbar_wait(wtready, (ci - 1) & 1, err);  // W^T of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16(tmem + CF::COL_P, kmaj(kt, kk), kmaj(qt, kk), id_p, kk > 0 ? 1u : 0u);
                mma_commit(pfull);
                if (ci > 0) {
                    ok = mbar_wait(dfree, (ci - 1) & 1, err);  // dV, dB of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    mma_bf16(tmem + CF::COL_D, kmaj(kt, kk), sdesc(gb + kk * 2048, kAtom, 1024), id_n,
                             kk > 0 ? 1u : 0u);
                    mma_bf16(tmem + CF::COL_D + kLane16, kmaj(vt, kk),
                             sdesc(gb + (kk / 4) * kAtom + (kk % 4) * 32, 16, 1024), id_t, kk > 0 ? 1u : 0u);
                }
                ok = mbar_wait(ptready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dV += P~^T GN
                    mma_bf16(tmem + CF::COL_D, sdesc(pta + kk * 32, 16, 1024), mnmaj(nt, kk), id_n, 1u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // W^T = V GN^T
                    mma_bf16(tmem + CF::COL_P, kmaj(vt, kk), kmaj(nt, kk), id_p, kk > 0 ? 1u : 0u);
                mma_commit(wfull);
                ok = mbar_wait(wtready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dB += W~^T A
                    mma_bf16(tmem + CF::COL_D + kLane16, sdesc(pta + kk * 32, 16, 1024), mnmaj(qt, kk), id_n, 1u);
                mma_commit(dfull);
                mma_commit(empty + s);
            }
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int a = sp * 32 + lane;  // the state row (d_k) this thread owns in TMEM
        seed_state_row(tmem + CF::COL_G + lane_base, tmem + CF::COL_H + lane_base,
                       suffix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D), a, normalize != 0, false);
        for (int ci = 0; ci < nci; ++ci) {
            const int c = chunk_of(ci);
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int valid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            mbar_wait(full + s, u & 1, err);
            if (mapped) {
                uint8_t* sg = sgn + s * CF::SGN;
                transform_tile<PHI, true>(st + kTile, et, C, false, sg, true);
                transform_tile<PHI, true>(st, et, C, false, sg, false);
            }
            // the chunk's gden: fp32 for the W~ mask, [hi; lo] rows for the h update
            if (et < C) {
                const float gd = (normalize && et < valid) ? gden_in[(size_t)bh * N + (size_t)c * C + et] : 0.f;
                gdf[(ci & 1) * C + et] = gd;
                if (normalize) {
                    const __nv_bfloat16 gh = __float2bfloat16_rn(gd);
                    const __nv_bfloat16 gl = __float2bfloat16_rn(gd - __bfloat162float(gh));
                    uint8_t* base = bgd + (ci & 1) * CF::BGD;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(0, et)) = gh;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(1, et)) = gl;
                }
            }
            if (ci > 0) {
                mbar_wait(gdone, (ci - 1) & 1, err);
                tc_fence_after();
            }
            // G_next -> bf16 operand [d_k][d_v]; h_next -> fp32
            state_row_to_bf16(tmem + CF::COL_G + lane_base, gbm + (ci & 1) * CF::BGM, a);
            float hv = 0.f;
            if (normalize) {
                uint32_t hr[2];
                tmem_ld2(tmem + CF::COL_H + lane_base, hr);
                tmem_ld_wait();
                hv = __uint_as_float(hr[0]) + __uint_as_float(hr[1]);
            }
            hf[(ci & 1) * D + a] = hv;
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);
        }
    } else {
        // ---------------- mask and epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int j = sp * 16 + (lane & 15);  // key row of the chunk
        const int half = lane >> 4;
        const int et2 = threadIdx.x - 192;
        bool ok = true;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = chunk_of(ci);
            const int s = ci % CF::STAGES;
            uint8_t* st = stages + s * CF::STAGE;
            // ---- P~^T: query i >= key j
            ok = mbar_wait(pfull, ci & 1, err) && ok;
            tc_fence_after();
            {
                uint32_t r[32];
                ld_half32(tmem + CF::COL_P + lane_base, r);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 32 * half + 8 * g + e;
                        f[e] = i >= j ? __uint_as_float(r[8 * g + e]) : 0.f;
                    }
                    *reinterpret_cast<uint4*>(pt + sw128_off(j, 32 * half + 8 * g)) = pack8(f);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ptready);
            // ---- W~^T = (W^T + gden_i) masked
            ok = ok && mbar_wait(wfull, ci & 1, err);
            tc_fence_after();
            {
                const float* gd = gdf + (ci & 1) * C;
                uint32_t r[32];
                ld_half32(tmem + CF::COL_P + lane_base, r);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 32 * half + 8 * g + e;
                        f[e] = i >= j ? __uint_as_float(r[8 * g + e]) + gd[i] : 0.f;
                    }
                    *reinterpret_cast<uint4*>(pt + sw128_off(j, 32 * half + 8 * g)) = pack8(f);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(wtready);
            // ---- dk = phi'(k) (dB + h_next), dv = dV over the K and V tiles
            ok = ok && mbar_wait(dfull, ci & 1, err);
            tc_fence_after();
            uint32_t dv[64], db[64];
            ld_half64(tmem + CF::COL_D + lane_base, dv);
            ld_half64(tmem + CF::COL_D + lane_base + kLane16, db);
            tc_fence_before();
            mbar_arrive(dfree);
            uint8_t* kt = st + kTile;
            uint8_t* vt = kt + kTile;
            const float* hb = hf + (ci & 1) * D;
            const uint8_t* sg = sgn + s * CF::SGN + j * 16;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                const int col = 64 * half + 8 * g;
                float fk[8], fv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    fk[e] = __uint_as_float(db[8 * g + e]) + hb[col + e];
                    fv[e] = __uint_as_float(dv[8 * g + e]);
                }
                uint4* pk = reinterpret_cast<uint4*>(kt + tile_off(j, col));
                times_phi_grad<PHI>(fk, PHI == PHI_RELU1 ? sg[col / 8] : 0u, *pk);
                *pk = pack8(fk);
                *reinterpret_cast<uint4*>(vt + tile_off(j, col)) = pack8(fv);
            }
            fence_async_smem();
            named_bar(3, 128);
            if (et2 == 0) {
                if (ok) {
                    store_tile(&mDk, kt, c * C, bh);
                    store_tile(&mDv, vt, c * C, bh);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(empty + s);
            }
        }
        if (et2 == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CF::TMEM_COLS);
    }
}

template <int PHI>
cudaError_t launch_kt(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                      const float* gden, const float* suffix, int block_tokens, int nblk, void* dk, void* dv,
                      uint32_t* err, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mgn, mdk, mdv;
    cudaError_t e = make_map(&mq, q, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mk, k, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mv, v, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mgn, gn, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mdk, dk, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mdv, dv, kD, p.N, p.bh(), kC);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_bwd_causal_kv_t_kernel<PHI>>(KtCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_bwd_causal_kv_t_kernel<PHI>, dim3(nblk, (unsigned)p.bh()), dim3(KtCfg::THREADS),
                      KtCfg::SMEM, st, mq, mk, mv, mgn, mdk, mdv, suffix, gden, p.N, block_tokens, nblk,
                      p.normalize, err);
}

template <int PHI>
cudaError_t launch_qt(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                      const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden, float* grec,
                      uint32_t* err, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mg, mgn, mdq;
    cudaError_t e = make_map(&mq, q, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mk, k, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mv, v, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mg, dout, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mgn, gn, kD, p.N, p.bh(), kC);
    if (e == cudaSuccess) e = make_map(&mdq, dq, kD, p.N, p.bh(), kC);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_bwd_causal_q_t_kernel<PHI>>(QtCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_bwd_causal_q_t_kernel<PHI>, dim3(nblk, (unsigned)p.bh()), dim3(QtCfg::THREADS), QtCfg::SMEM,
                      st, mq, mk, mv, mg, mgn, mdq, prefix, p.N, block_tokens, nblk, p.normalize, gden, grec, err);
}

}  // namespace

cudaError_t tc_causal_backward_q_t(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                   const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden,
                                   float* grec, uint32_t* err, cudaStream_t st) {
    if (p.d != kD || p.dtype != DT_BF16 || block_tokens % kC != 0) return cudaErrorInvalidValue;
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1:
            return launch_qt<PHI_RELU1>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err, st);
        case PHI_ELU1:
            return launch_qt<PHI_ELU1>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err, st);
        default:
            return launch_qt<PHI_IDENTITY>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err,
                                           st);
    }
}

cudaError_t tc_causal_backward_kv_t(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                                    const float* gden, const float* suffix, int block_tokens, int nblk, void* dk,
                                    void* dv, uint32_t* err, cudaStream_t st) {
    if (p.d != kD || p.dtype != DT_BF16 || block_tokens % kC != 0) return cudaErrorInvalidValue;
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1:
            return launch_kt<PHI_RELU1>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
        case PHI_ELU1:
            return launch_kt<PHI_ELU1>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
        default:
            return launch_kt<PHI_IDENTITY>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
    }
}

}  // namespace la
