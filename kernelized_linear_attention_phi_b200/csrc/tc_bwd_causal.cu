// Gradients of the causal form, first sweep, on tcgen05 tensor cores (bf16,
// d = 64, 64-token chunks): dq, the scaled upstream gradient gn (bf16) and
// gden (fp32) for the second sweep, and per block the (G, h) record of its
// chunks (summed from the end by the block-state scan).
//
// With a = phi(q), b = phi(k), g = dL/dout, w_ij = a_i . b_j for j <= i:
//   den_i = sum_j w_ij, out_i = sum_j w_ij v_j / den_i,
//   gn_i = g_i / den_i, gden_i = -(g_i . out_i) / den_i,
//   dq_i = phi'(q_i) * sum_{j <= i} (gn_i . v_j + gden_i) b_j
//   G = sum_i a_i gn_i^T, h = sum_i a_i gden_i over the block's queries.
// One CTA per (block, head) sweeps the block's chunks in order with the
// running state S (fp32, M = d_k) and z of the keys before the chunk in
// TMEM, seeded from the block's prefix record. For chunk c (A, B, V, GN the
// chunk's rows):
//   S_prev, z_prev -> bf16 operands                           [prep]
//   S += B^T V, z += B^T 1                                     [MMA]
//   P = A B^T -> P~ (j <= i, bf16), rowsum                     [MMA, mask]
//   O = A S_prev + P~ V, den = rowsum + A [z_hi; z_lo]         [MMA]
//   out, gn (over the dO tile, then stored), gden              [epilogue]
//   dA = GN S_prev^T (the S_prev operand read K-major)         [MMA]
//   W = GN V^T -> W~ = (W + gden 1^T) masked (bf16)            [MMA, mask]
//   G += A^T GN, h += A^T [gden_hi; gden_lo]                    [MMA]
//   dA += W~ B; dq = phi'(q) (dA + gden z_prev)                [MMA, epilogue]
// The chunk's M = 64 accumulators pair up in the two 16-lane halves of each
// TMEM sub-partition: S / G, z / h and O / dA share columns.
//
// Warp roles (320 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer,
// warps 2-5 prep (phi on the Q and K tiles, relu'(q) bits, state ->
// operands), warps 6-9 masks and epilogues (row i = 16 sp + (lane & 15), the
// warp halves take the two 32-column halves).

#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

struct CqCfg {
    static constexpr int D = 64, C = 64;
    static constexpr int TILE = C * D * 2;    // one [64 x 64] bf16 tile
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 4 * TILE;    // Q, K, V, dO (gn, then dq)
    static constexpr int B3 = D * D * 2;      // S_prev bf16 [d_k][d_v] (x2)
    static constexpr int BZ = 16 * D * 2;     // [z_hi; z_lo; 0] (x2)
    static constexpr int ONES = 16 * C * 2;   // all-ones [16][C], K-major
    static constexpr int PT = C * C * 2;      // P~, then W~ [query][key], K-major
    static constexpr int BGD = 16 * C * 2;    // [gden_hi; gden_lo; 0] over the chunk, K-major
    static constexpr int SGN = C * D / 8;     // relu'(q) bits (x STAGES)
    static constexpr int ZF = 2 * D * 4;      // z_prev fp32 (x2)
    static constexpr uint32_t LANE16 = 16u << 16;
    // TMEM columns (M = 64 accumulators: lanes 0..15 and 16..31 of each sub-partition)
    static constexpr int COL_S = 0;      // S (lanes 0-15), G (lanes 16-31)
    static constexpr int COL_Z = 64;     // z, h
    static constexpr int COL_P = 80;     // P, then W
    static constexpr int COL_O = 144;    // O (lanes 0-15), dA (lanes 16-31)
    static constexpr int COL_OZ = 208;   // den terms
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr int NBAR = 2 * STAGES + 11;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * B3 + 2 * BZ + ONES + PT + BGD + STAGES * SGN +
                                   ZF + 8 * NBAR + 16;
    static constexpr int THREADS = 320;
    static_assert(COL_OZ + 16 <= (int)TMEM_COLS, "TMEM");
    // two resident CTAs per SM: 228 KiB per SM, 1 KiB reserved per CTA
    static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
};

template <int PHI>
__global__ void __launch_bounds__(CqCfg::THREADS, 2)
tc_bwd_causal_q_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                       const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mGo,
                       const __grid_constant__ CUtensorMap mGn, const __grid_constant__ CUtensorMap mDq,
                       const float* __restrict__ prefix, int N, int block_tokens, int nblk, int normalize,
                       float* __restrict__ gden_out, float* __restrict__ grec, uint32_t* __restrict__ err) {
    using CF = CqCfg;
    constexpr int D = CF::D, C = CF::C;
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
                tma_load_3d(st, &mQ, full + s, 0, row, bh);
                tma_load_3d(st + CF::TILE, &mK, full + s, 0, row, bh);
                tma_load_3d(st + 2 * CF::TILE, &mV, full + s, 0, row, bh);
                tma_load_3d(st + 3 * CF::TILE, &mGo, full + s, 0, row, bh);
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
            bool ok = true;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t qt = smem_u32(stages + s * CF::STAGE), kt = qt + CF::TILE, vt = kt + CF::TILE,
                               gt = vt + CF::TILE;
                const uint32_t b3a = smem_u32(b3 + (ci & 1) * CF::B3), bza = smem_u32(bz + (ci & 1) * CF::BZ);
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t a = sdesc(kt + kk * 2048, C * 128, 1024);  // B^T, MN-major
                    mma_bf16(tmem + CF::COL_S, a, sdesc(vt + kk * 2048, C * 128, 1024), id_s, 1u);
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
                    mma_bf16(tmem + CF::COL_P, sdesc(qt + kk * 32, 16, 1024), sdesc(kt + kk * 32, 16, 1024), id_p,
                             kk > 0 ? 1u : 0u);
                mma_commit(pfull);
                if (ci > 0) {
                    ok = mbar_wait(gnready, (ci - 1) & 1, err);  // O of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = sdesc(qt + kk * 32, 16, 1024);
                    mma_bf16(tmem + CF::COL_O, a, sdesc(b3a + kk * 2048, D * 128, 1024), id_o, kk > 0 ? 1u : 0u);
                    if (normalize)
                        mma_bf16(tmem + CF::COL_OZ, a, sdesc(bza + kk * 32, 16, 1024), id_oz, kk > 0 ? 1u : 0u);
                }
                ok = mbar_wait(ptready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)
                    mma_bf16(tmem + CF::COL_O, sdesc(pta + kk * 32, 16, 1024), sdesc(vt + kk * 2048, C * 128, 1024),
                             id_o, 1u);
                mma_commit(ofull);
                ok = mbar_wait(gnready, ci & 1, err);
                if (ok && ci > 0) ok = mbar_wait(dafree, (ci - 1) & 1, err);  // dA of the last chunk read
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // dA = GN S_prev^T
                    mma_bf16(tmem + CF::COL_O + CF::LANE16, sdesc(gt + kk * 32, 16, 1024), sdesc(b3a + kk * 32, 16, 1024),
                             id_a, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // W = GN V^T
                    mma_bf16(tmem + CF::COL_P, sdesc(gt + kk * 32, 16, 1024), sdesc(vt + kk * 32, 16, 1024), id_p,
                             kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {  // G += A^T GN, h += A^T [gden]
                    const uint64_t a = sdesc(qt + kk * 2048, C * 128, 1024);
                    const uint32_t accum = (ci == 0 && kk == 0) ? 0u : 1u;
                    mma_bf16(tmem + CF::COL_S + CF::LANE16, a, sdesc(gt + kk * 2048, C * 128, 1024), id_s, accum);
                    if (normalize) mma_bf16(tmem + CF::COL_Z + CF::LANE16, a, sdesc(gda + kk * 32, 16, 1024), id_z, accum);
                }
                mma_commit(wfull);
                ok = mbar_wait(wtready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dA += W~ B
                    mma_bf16(tmem + CF::COL_O + CF::LANE16, sdesc(pta + kk * 32, 16, 1024),
                             sdesc(kt + kk * 2048, C * 128, 1024), id_o, 1u);
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
        const float* pre = prefix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
        {
            // seed S, z with the block's prefix: row 16 sp + lane (lanes 0..15)
            const int a = sp * 16 + lane;
            const bool own = lane < 16;
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
        // No early exit in this warpgroup: after a failed wait the loop runs
        // on without waiting (see cta_abort).
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int kvalid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            mbar_wait(full + s, u & 1, err);
            uint4* qt = reinterpret_cast<uint4*>(st);
            uint4* kt = reinterpret_cast<uint4*>(st + CF::TILE);
            uint8_t* sg = sgn + s * CF::SGN;
            uint4 kx[4], qx[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                kx[j] = kt[et + 128 * j];
                if (mapped) qx[j] = qt[et + 128 * j];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int p = et + 128 * j, r = p >> 3;
                kt[p] = r < kvalid ? phi8<PHI>(kx[j]) : make_uint4(0, 0, 0, 0);  // keys past N stay zero
                if (mapped) {
                    if (PHI == PHI_RELU1) sg[r * 8 + ((p & 7) ^ (r & 7))] = static_cast<uint8_t>(positive_bits(qx[j]));
                    qt[p] = phi8<PHI>(qx[j]);
                }
            }
            if (ci > 0) {
                mbar_wait(bsdone, (ci - 1) & 1, err);
                tc_fence_after();
            }
            // S_prev -> bf16 MN-major operand [d_k][d_v]
            uint8_t* b3b = b3 + (ci & 1) * CF::B3;
            {
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
            // z_prev -> rows 0 (hi) and 1 (lo) of the z operand, and in fp32 for the dq epilogue
            if (normalize) {
                uint32_t r[16];
                tmem_ld16(tmem + CF::COL_Z + lane_base, r);
                tmem_ld_wait();
                if (lane < 16) {
                    const int a = sp * 16 + lane;
                    const float zv = __uint_as_float(r[0]);
                    const __nv_bfloat16 zh = __float2bfloat16_rn(zv);
                    const __nv_bfloat16 zl = __float2bfloat16_rn(zv - __bfloat162float(zh));
                    uint8_t* base = bz + (ci & 1) * CF::BZ;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(0, a)) = zh;
                    *reinterpret_cast<__nv_bfloat16*>(base + sw128_off(1, a)) = zl;
                    zf[(ci & 1) * D + a] = zv;
                }
            } else if (lane < 16) {
                zf[(ci & 1) * D + sp * 16 + lane] = 0.f;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);
        }
    } else {
        // ---------------- mask and epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int i = sp * 16 + (lane & 15);  // query row of the chunk
        const int half = lane >> 4;           // this thread's 32-column half
        const int et2 = threadIdx.x - 192;
        // No early exit in this warpgroup (named barrier 3); a failed wait
        // only suppresses the stores.
        bool ok = true;
        // row i of the P / W accumulator, this half's columns
        auto ld_row = [&](uint32_t col, uint32_t (&r)[32]) {
            tmem_ld16x2<32>(tmem + col + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
            tmem_ld16x2<32>(tmem + col + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
            tmem_ld_wait();
        };
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES;
            const int valid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            uint8_t* gt = st + 3 * CF::TILE;  // dO: g, then gn, then dq
            // ---- P~ = P masked (key j <= query i), row sums
            ok = mbar_wait(pfull, ci & 1, err) && ok;
            tc_fence_after();
            float rs = 0.f;
            {
                uint32_t r[32];
                ld_row(CF::COL_P, r);
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
            uint32_t o[32];
            ld_row(CF::COL_O, o);
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
            for (int g = 0; g < 4; ++g) {
                uint4* p = reinterpret_cast<uint4*>(gt + sw128_off(i, 32 * half + 8 * g));
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
                tma_store_3d(&mGn, gt, 0, c * C, bh);
                bulk_commit();
            }
            // ---- W~ = (W + gden_i) masked (key j <= query i)
            ok = ok && mbar_wait(wfull, ci & 1, err);
            tc_fence_after();
            {
                uint32_t r[32];
                ld_row(CF::COL_P, r);
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
            uint32_t a[32];
            ld_row(CF::COL_O + CF::LANE16, a);
            tc_fence_before();
            mbar_arrive(dafree);
            if (et2 == 0) bulk_wait_read0();  // the gn store has read the tile
            named_bar(3, 128);
            const float* zb = zf + (ci & 1) * D;
            const uint8_t* sg = sgn + s * CF::SGN + i * 8;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int col = 32 * half + 8 * g;
                float f[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(a[8 * g + e]) + gden * zb[col + e];
                const uint4 pq = PHI == PHI_ELU1 ? *reinterpret_cast<const uint4*>(st + sw128_off(i, col))
                                                 : make_uint4(0, 0, 0, 0);
                times_phi_grad<PHI>(f, PHI == PHI_RELU1 ? sg[col / 8] : 0u, pq);
                *reinterpret_cast<uint4*>(gt + sw128_off(i, col)) = pack8(f);
            }
            fence_async_smem();
            named_bar(3, 128);
            if (et2 == 0) {
                if (ok) {
                    tma_store_3d(&mDq, gt, 0, c * C, bh);
                    bulk_commit();
                    bulk_wait_read0();
                }
                mbar_arrive(empty + s);
            }
        }
        // ---- the block's (G, h): G in lanes 16..31 of the S columns, h of the z columns
        ok = ok && mbar_wait(gfull, 0, err);
        tc_fence_after();
        {
            float* rec = grec + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
            uint32_t v[32];
            ld_row(CF::COL_S + CF::LANE16, v);
            uint32_t hr[2] = {0u, 0u};
            if (normalize) {
                tmem_ld2(tmem + CF::COL_Z + lane_base, hr);  // lanes 16..31: h of row i
                tmem_ld_wait();
            }
            float4* o4 = reinterpret_cast<float4*>(rec + (size_t)i * D + 32 * half);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
                o4[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                     __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
            if (half == 1) rec[(size_t)D * D + i] = __uint_as_float(hr[0]) + __uint_as_float(hr[1]);
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
// One CTA per (block, head) sweeps the block's chunks from the last to the
// first with the running state G (fp32, M = d_k) and h of the queries after
// the chunk in TMEM, seeded from the block's suffix record. For chunk c (keys
// j and queries i its rows; A = phi(Q), B = phi(K), GN from the first sweep):
//   G_next, h_next -> bf16 operand, fp32 copy                  [prep]
//   G += A^T GN, h += A^T [gden_hi; gden_lo]                   [MMA]
//   P^T = B A^T -> P~^T (i >= j, bf16)                         [MMA, mask]
//   dV = B G_next + P~^T GN;  dB = V G_next^T                  [MMA]
//   W^T = V GN^T -> W~^T = (W^T + 1 gden^T) masked (bf16)       [MMA, mask]
//   dB += W~^T A;  dk = phi'(k) (dB + h_next), dv = dV         [MMA, epilogue]
// dV and dB pair up in the two 16-lane halves of the same TMEM columns.
struct CkCfg {
    static constexpr int D = 64, C = 64;
    static constexpr int TILE = C * D * 2;
    static constexpr int STAGES = 2;
    static constexpr int STAGE = 4 * TILE;    // Q, K, V, GN (K, V then dk, dv)
    static constexpr int BGM = D * D * 2;     // G_next bf16 [d_k][d_v] (x2)
    static constexpr int PT = C * C * 2;      // P~^T, then W~^T [key][query], K-major
    static constexpr int BGD = 16 * C * 2;    // [gden_hi; gden_lo; 0] over the chunk (x2)
    static constexpr int SGN = C * D / 8;     // relu'(k) bits (x STAGES)
    static constexpr int VEC = 2 * D * 4;     // h_next and the chunk's gden, fp32 (x2 each)
    static constexpr uint32_t LANE16 = 16u << 16;
    static constexpr int COL_G = 0;    // G (lanes 0-15)
    static constexpr int COL_H = 64;   // h
    static constexpr int COL_P = 80;   // P^T, then W^T
    static constexpr int COL_D = 144;  // dV (lanes 0-15), dB (lanes 16-31)
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr int NBAR = 2 * STAGES + 9;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * BGM + PT + 2 * BGD + STAGES * SGN + 2 * VEC +
                                   8 * NBAR + 16;
    static constexpr int THREADS = 320;
    static_assert(COL_D + 64 <= (int)TMEM_COLS, "TMEM");
    static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
};

template <int PHI>
__global__ void __launch_bounds__(CkCfg::THREADS, 2)
tc_bwd_causal_kv_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                        const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mGn,
                        const __grid_constant__ CUtensorMap mDk, const __grid_constant__ CUtensorMap mDv,
                        const float* __restrict__ suffix, const float* __restrict__ gden_in, int N,
                        int block_tokens, int nblk, int normalize, uint32_t* __restrict__ err) {
    using CF = CkCfg;
    constexpr int D = CF::D, C = CF::C;
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
                tma_load_3d(st, &mQ, full + s, 0, row, bh);
                tma_load_3d(st + CF::TILE, &mK, full + s, 0, row, bh);
                tma_load_3d(st + 2 * CF::TILE, &mV, full + s, 0, row, bh);
                tma_load_3d(st + 3 * CF::TILE, &mGn, full + s, 0, row, bh);
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
            bool ok = true;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t qt = smem_u32(stages + s * CF::STAGE), kt = qt + CF::TILE, vt = kt + CF::TILE,
                               nt = vt + CF::TILE;
                const uint32_t gb = smem_u32(gbm + (ci & 1) * CF::BGM), gda = smem_u32(bgd + (ci & 1) * CF::BGD);
                ok = mbar_wait(bprep, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk) {
                    const uint64_t a = sdesc(qt + kk * 2048, C * 128, 1024);  // A^T, MN-major
                    mma_bf16(tmem + CF::COL_G, a, sdesc(nt + kk * 2048, C * 128, 1024), id_g, 1u);
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
                    mma_bf16(tmem + CF::COL_P, sdesc(kt + kk * 32, 16, 1024), sdesc(qt + kk * 32, 16, 1024), id_p,
                             kk > 0 ? 1u : 0u);
                mma_commit(pfull);
                if (ci > 0) {
                    ok = mbar_wait(dfree, (ci - 1) & 1, err);  // dV, dB of the last chunk read
                    if (!ok) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    mma_bf16(tmem + CF::COL_D, sdesc(kt + kk * 32, 16, 1024), sdesc(gb + kk * 2048, D * 128, 1024),
                             id_n, kk > 0 ? 1u : 0u);
                    mma_bf16(tmem + CF::COL_D + CF::LANE16, sdesc(vt + kk * 32, 16, 1024),
                             sdesc(gb + kk * 32, 16, 1024), id_t, kk > 0 ? 1u : 0u);
                }
                ok = mbar_wait(ptready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dV += P~^T GN
                    mma_bf16(tmem + CF::COL_D, sdesc(pta + kk * 32, 16, 1024), sdesc(nt + kk * 2048, C * 128, 1024),
                             id_n, 1u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // W^T = V GN^T
                    mma_bf16(tmem + CF::COL_P, sdesc(vt + kk * 32, 16, 1024), sdesc(nt + kk * 32, 16, 1024), id_p,
                             kk > 0 ? 1u : 0u);
                mma_commit(wfull);
                ok = mbar_wait(wtready, ci & 1, err);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < C / 16; ++kk)  // dB += W~^T A
                    mma_bf16(tmem + CF::COL_D + CF::LANE16, sdesc(pta + kk * 32, 16, 1024),
                             sdesc(qt + kk * 2048, C * 128, 1024), id_n, 1u);
                mma_commit(dfull);
                mma_commit(empty + s);
            }
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const float* suf = suffix + ((size_t)bh * nblk + blk) * (size_t)(D * D + D);
        {
            // seed G, h with the block's suffix: row 16 sp + lane (lanes 0..15)
            const int a = sp * 16 + lane;
            const bool own = lane < 16;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t r[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 x = own ? reinterpret_cast<const float4*>(suf + (size_t)a * D + c0)[q4]
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    r[4 * q4] = __float_as_uint(x.x);
                    r[4 * q4 + 1] = __float_as_uint(x.y);
                    r[4 * q4 + 2] = __float_as_uint(x.z);
                    r[4 * q4 + 3] = __float_as_uint(x.w);
                }
                tmem_st16(tmem + CF::COL_G + lane_base + c0, r);
            }
            uint32_t r[16];
            const uint32_t hv = (own && normalize) ? __float_as_uint(suf[(size_t)D * D + a]) : 0u;
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = hv;
            tmem_st16(tmem + CF::COL_H + lane_base, r);
            tmem_st_wait();
        }
        for (int ci = 0; ci < nci; ++ci) {
            const int c = chunk_of(ci);
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int valid = min(C, N - c * C);
            uint8_t* st = stages + s * CF::STAGE;
            mbar_wait(full + s, u & 1, err);
            if (mapped) {
                uint4* qt = reinterpret_cast<uint4*>(st);
                uint4* kt = reinterpret_cast<uint4*>(st + CF::TILE);
                uint8_t* sg = sgn + s * CF::SGN;
                uint4 kx[4], qx[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    kx[j] = kt[et + 128 * j];
                    qx[j] = qt[et + 128 * j];
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int p = et + 128 * j, r = p >> 3;
                    if (PHI == PHI_RELU1) sg[r * 8 + ((p & 7) ^ (r & 7))] = static_cast<uint8_t>(positive_bits(kx[j]));
                    kt[p] = phi8<PHI>(kx[j]);
                    qt[p] = phi8<PHI>(qx[j]);
                }
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
            {
                const int a = sp * 16 + (lane & 15);
                const int cb = lane < 16 ? 0 : 32;
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + CF::COL_G + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + CF::COL_G + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                uint32_t hr[16];
                tmem_ld16(tmem + CF::COL_H + lane_base, hr);
                tmem_ld_wait();
                uint8_t* gbb = gbm + (ci & 1) * CF::BGM;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * g + e]);
                    *reinterpret_cast<uint4*>(gbb + sw128_off(a, cb + 8 * g)) = pack8(f);
                }
                if (lane < 16) hf[(ci & 1) * D + a] = normalize ? __uint_as_float(hr[0]) : 0.f;
            }
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
        auto ld_row = [&](uint32_t col, uint32_t (&r)[32]) {
            tmem_ld16x2<32>(tmem + col + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
            tmem_ld16x2<32>(tmem + col + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
            tmem_ld_wait();
        };
        for (int ci = 0; ci < nci; ++ci) {
            const int c = chunk_of(ci);
            const int s = ci % CF::STAGES;
            uint8_t* st = stages + s * CF::STAGE;
            // ---- P~^T: query i >= key j
            ok = mbar_wait(pfull, ci & 1, err) && ok;
            tc_fence_after();
            {
                uint32_t r[32];
                ld_row(CF::COL_P, r);
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
                ld_row(CF::COL_P, r);
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
            uint32_t dv[32], db[32];
            ld_row(CF::COL_D, dv);
            ld_row(CF::COL_D + CF::LANE16, db);
            tc_fence_before();
            mbar_arrive(dfree);
            uint8_t* kt = st + CF::TILE;
            uint8_t* vt = kt + CF::TILE;
            const float* hb = hf + (ci & 1) * D;
            const uint8_t* sg = sgn + s * CF::SGN + j * 8;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const int col = 32 * half + 8 * g;
                float fk[8], fv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    fk[e] = __uint_as_float(db[8 * g + e]) + hb[col + e];
                    fv[e] = __uint_as_float(dv[8 * g + e]);
                }
                uint4* pk = reinterpret_cast<uint4*>(kt + sw128_off(j, col));
                times_phi_grad<PHI>(fk, PHI == PHI_RELU1 ? sg[col / 8] : 0u, *pk);
                *pk = pack8(fk);
                *reinterpret_cast<uint4*>(vt + sw128_off(j, col)) = pack8(fv);
            }
            fence_async_smem();
            named_bar(3, 128);
            if (et2 == 0) {
                if (ok) {
                    tma_store_3d(&mDk, kt, 0, c * C, bh);
                    tma_store_3d(&mDv, vt, 0, c * C, bh);
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
cudaError_t launch_ck(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                      const float* gden, const float* suffix, int block_tokens, int nblk, void* dk, void* dv,
                      uint32_t* err, cudaStream_t st) {
    constexpr int C = CkCfg::C, D = CkCfg::D;
    CUtensorMap mq, mk, mv, mgn, mdk, mdv;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mk, k, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mgn, gn, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mdk, dk, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mdv, dv, D, p.N, p.bh(), C);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_bwd_causal_kv_kernel<PHI>>(CkCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_bwd_causal_kv_kernel<PHI>, dim3(nblk, (unsigned)p.bh()), dim3(CkCfg::THREADS),
                      CkCfg::SMEM, st, mq, mk, mv, mgn, mdk, mdv, suffix, gden, p.N, block_tokens, nblk,
                      p.normalize, err);
}

template <int PHI>
cudaError_t launch_cq(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                      const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden, float* grec,
                      uint32_t* err, cudaStream_t st) {
    constexpr int C = CqCfg::C, D = CqCfg::D;
    CUtensorMap mq, mk, mv, mg, mgn, mdq;
    cudaError_t e = make_map(&mq, q, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mk, k, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mv, v, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mg, dout, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mgn, gn, D, p.N, p.bh(), C);
    if (e == cudaSuccess) e = make_map(&mdq, dq, D, p.N, p.bh(), C);
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_bwd_causal_q_kernel<PHI>>(CqCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(tc_bwd_causal_q_kernel<PHI>, dim3(nblk, (unsigned)p.bh()), dim3(CqCfg::THREADS), CqCfg::SMEM,
                      st, mq, mk, mv, mg, mgn, mdq, prefix, p.N, block_tokens, nblk, p.normalize, gden, grec, err);
}

}  // namespace

bool tc_causal_backward_supported(const Problem& p, int block_tokens) {
    return p.dtype == DT_BF16 && (p.d == 64 || p.d == 128) && block_tokens % CqCfg::C == 0;
}

cudaError_t tc_causal_backward_q(const Problem& p, const void* q, const void* k, const void* v, const void* dout,
                                 const float* prefix, int block_tokens, int nblk, void* dq, void* gn, float* gden,
                                 float* grec, uint32_t* err, cudaStream_t st) {
    if (!tc_causal_backward_supported(p, block_tokens)) return cudaErrorInvalidValue;
    if (p.d == 128)
        return tc_causal_backward_q_t(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err, st);
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1:
            return launch_cq<PHI_RELU1>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err, st);
        case PHI_ELU1:
            return launch_cq<PHI_ELU1>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err, st);
        default:
            return launch_cq<PHI_IDENTITY>(p, q, k, v, dout, prefix, block_tokens, nblk, dq, gn, gden, grec, err,
                                           st);
    }
}

cudaError_t tc_causal_backward_kv(const Problem& p, const void* q, const void* k, const void* v, const void* gn,
                                  const float* gden, const float* suffix, int block_tokens, int nblk, void* dk,
                                  void* dv, uint32_t* err, cudaStream_t st) {
    if (!tc_causal_backward_supported(p, block_tokens)) return cudaErrorInvalidValue;
    if (p.d == 128)
        return tc_causal_backward_kv_t(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1:
            return launch_ck<PHI_RELU1>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
        case PHI_ELU1:
            return launch_ck<PHI_ELU1>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
        default:
            return launch_ck<PHI_IDENTITY>(p, q, k, v, gn, gden, suffix, block_tokens, nblk, dk, dv, err, st);
    }
}

}  // namespace la
