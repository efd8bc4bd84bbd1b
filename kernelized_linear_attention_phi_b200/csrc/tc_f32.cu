// fp32 linear attention (d = 64) on tcgen05 tensor cores with split bf16
// operands.
//
// Every fp32 operand x enters the tensor core as two bf16 values, hi =
// bf16(x) and lo = bf16(x - hi), which together hold x to within 2^-16 |x|,
// and every product is accumulated in fp32 in TMEM as hi*hi + hi*lo + lo*hi:
// three bf16 MMAs where the bf16 kernels issue one. The dropped lo*lo term
// and the split's remainder keep a product within about 3 * 2^-16 of its
// exact value, and the outputs within about 1e-5 of the exact ones (largest
// relative row error), inside the fp32 tolerance of 1e-4.
//
// The fp32 tiles land by TMA (two 32-column boxes, 128-byte swizzle); the prep
// warps read a tile into registers and rewrite the same 16 KB as its hi and lo
// bf16 tiles (phi applied first), in the layout the bf16 kernels' TMA writes.
// z is summed on the CUDA cores in fp32 (column sums of the transformed K
// tiles); phi(Q).z rides on the state product: the hi state operand carries
// z's three bf16 parts (hi, mid, lo: all 24 bits of z) as extra columns 64..66
// (N = 80), so O's columns 64..66 hold phi(Q).z. One kernel, three modes:
//   kState    the state (S, z) of one block of keys, written as one record
//             (S [d_k][d_v] then z): block states of the chunked forms and
//             the split-N partials of the KV summary
//   kSweep    causal outputs of one block from its prefix record: the chunked
//             algorithm of the bf16 d = 64 sweep (tc_sweep.cu), products split
//   kReadout  non-causal outputs from a head's total state:
//             out_i = phi(Q_i) S / phi(Q_i).z (S alone when unnormalized)
//   kGather   the prefix mask: kSweep over chunk c with the queries whose
//             bin floor((m_i + 1) / 64) is c gathered by TMA tile::gather4
//             into a ring of query slots, each row's keys limited to m_i
// Warp roles (320 threads) as in the bf16 sweep: warp 0 TMA, warp 1 MMA +
// TMEM, warps 2-5 prep (phi, splits, z, state -> operands), warps 6-9 mask
// (P~ split, denominators, epilogue; in kState the final record of S).

#include <algorithm>

#include "device.h"
#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

enum { kState = 0, kSweep = 1, kReadout = 2, kGather = 3 };

template <int MODE>
struct F32Cfg {
    static constexpr int D = 64, C = 64;
    static constexpr bool GATHER = MODE == kGather;
    static constexpr bool SWEEP = MODE == kSweep || MODE == kGather;  // the chunked sweep
    static constexpr bool HAS_Q = MODE == kSweep || MODE == kReadout;  // Q tiles in the stage
    static constexpr bool HAS_KV = MODE != kReadout;
    static constexpr bool OUT = MODE != kState;
    static constexpr int FT = C * D * 4;   // one fp32 [C x D] tile; after prep its hi and lo bf16 tiles
    static constexpr int LO = C * D * 2;   // offset of the lo tile within it
    static constexpr int NT = (HAS_Q ? 1 : 0) + (HAS_KV ? 2 : 0);
    static constexpr int OFF_K = HAS_Q ? FT : 0;
    static constexpr int OFF_V = OFF_K + FT;
    // pipeline depth: the sweep's shared memory allows two stages; the state
    // and readout passes keep more tiles in flight at two CTAs per SM
    static constexpr int STAGES = SWEEP ? 2 : MODE == kState ? 3 : 4;
    static constexpr int MIN_BLOCKS = SWEEP ? 1 : 2;
    static constexpr int STAGE = NT * FT;
    static constexpr int PT = SWEEP ? 2 * C * C * 2 : 0;  // P~ hi and lo of one slot (x2 slots)
    static constexpr int NB3 = SWEEP ? 2 : MODE == kReadout ? 1 : 0;
    // state operands, MN-major [d_k][d_v]: hi (N = 80: 64 columns of S, then
    // an atom whose columns 0..2 are z hi / mid / lo and 3..15 zero), lo
    static constexpr int ATOM = D * D * 2;    // one [64 x 64] bf16 swizzle atom
    static constexpr int B3 = 3 * ATOM;       // S hi, z atom, S lo
    static constexpr int QS = GATHER ? 3 : 1;                // gathered query slots
    static constexpr int QG = GATHER ? QS * FT : 0;          // gathered fp32 queries, split in place
    static constexpr int ROWS = GATHER ? QS * 2 * C * 4 : 0;  // token / key limit per row, per query slot
    static constexpr int STG = (OUT && !GATHER) ? C * D * 4 : 0;  // fp32 output staging (two 32-column boxes)
    static constexpr int RED = HAS_KV ? 2 * 4 * D * 4 : 0;  // z column-sum partials [parity][warp][d]
    static constexpr int NBAR = 3 * STAGES + 1 + 4 * 2 + 3 * QS;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 2 * PT + NB3 * B3 + QG + STG + ROWS + RED +
                                   8 * NBAR + 16;
    // TMEM: M = 64 accumulators (rows in lanes 0..15 of each sub-partition);
    // the two slots of P and O share columns, slot 1 in lanes 16..31. O has
    // 80 columns: the outputs, then phi(Q).z hi / mid / lo in 64..66.
    static constexpr int COL_S = 0;
    static constexpr int COL_P = SWEEP ? 64 : 0;
    static constexpr int COL_O = SWEEP ? 128 : 0;
    static constexpr int COL_OZ = COL_O + D;
    static constexpr uint32_t TMEM_COLS = SWEEP ? 256u : MODE == kReadout ? 128u : 64u;
    static constexpr int THREADS = 320;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    // 228 KiB per SM, 1 KiB reserved per CTA; TMEM columns of all resident CTAs
    static_assert(MIN_BLOCKS * (SMEM + 1024) <= 228 * 1024 && MIN_BLOCKS * TMEM_COLS <= 512, "CTAs per SM");
    static_assert(STAGE % 1024 == 0 && FT % 1024 == 0, "1024-byte aligned operand tiles");
};

__device__ __forceinline__ uint32_t slot_lanes(int j) { return (uint32_t)j * (16u << 16); }

// hi / lo bf16 split of eight fp32 values
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo) {
    float h[8], l[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        h[e] = __bfloat162float(__float2bfloat16_rn(f[e]));
        l[e] = f[e] - h[e];
    }
    hi = pack8(h);
    lo = pack8(l);
}

// The prep warps' in-place rewrite of one fp32 tile at `tb` (two [C x 32]
// fp32 boxes, 128-byte swizzle) as its hi tile (tb) and lo tile (tb + LO),
// each [C x 64] bf16 with the 128-byte swizzle. Thread et takes column group
// g = et % 8 (columns 8g .. 8g + 7) of rows et / 8 + 16 i, i < 4. With phi,
// phi is applied first; rows at or beyond `valid` become 0. `colsum`, when
// given, receives this thread's sums of its 8 columns over its 4 rows (after
// phi and the row mask). Every prep thread calls it: it holds named barrier 2
// between the reads and the writes.
template <int PHI, bool APPLY>
__device__ __forceinline__ void split_tile(uint8_t* tb, int et, int valid, float* colsum) {
    constexpr int LO = 64 * 64 * 2;
    const int g = et & 7, box = g >> 2, j0 = 2 * (g & 3);
    float f[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = (et >> 3) + 16 * i;
        const uint8_t* rowp = tb + box * 8192 + r * 128;
        const float4 a = *reinterpret_cast<const float4*>(rowp + ((j0 ^ (r & 7)) << 4));
        const float4 b = *reinterpret_cast<const float4*>(rowp + (((j0 + 1) ^ (r & 7)) << 4));
        f[i][0] = a.x; f[i][1] = a.y; f[i][2] = a.z; f[i][3] = a.w;
        f[i][4] = b.x; f[i][5] = b.y; f[i][6] = b.z; f[i][7] = b.w;
    }
    named_bar(2, 128);  // every prep thread has read the tile
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = (et >> 3) + 16 * i;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            float x = f[i][e];
            if (APPLY) x = phi_apply(x, PHI);
            f[i][e] = r < valid ? x : 0.f;
            if (colsum != nullptr) colsum[e] += f[i][e];
        }
        uint4 hi, lo;
        split8(f[i], hi, lo);
        *reinterpret_cast<uint4*>(tb + sw128_off(r, 8 * g)) = hi;
        *reinterpret_cast<uint4*>(tb + LO + sw128_off(r, 8 * g)) = lo;
    }
}

// Thirty-two fp32 values of state row a (columns c0 .. c0 + 31) into the hi
// and lo MN-major operand tiles of the state operands at b3 (hi in atom 0, lo
// in atom 2).
__device__ __forceinline__ void split_state_row(uint8_t* b3, int a, int c0, const float* f) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        uint4 hi, lo;
        split8(f + 8 * g, hi, lo);
        *reinterpret_cast<uint4*>(b3 + sw128_off(a, c0 + 8 * g)) = hi;
        *reinterpret_cast<uint4*>(b3 + 2 * 64 * 64 * 2 + sw128_off(a, c0 + 8 * g)) = lo;
    }
}

// z (entry d_k) as its hi, mid, lo bf16 parts into columns 0, 1, 2 of row d_k
// of the z atom (atom 1 of the state operands at b3).
__device__ __forceinline__ void split_z(uint8_t* b3, int dk, float zv) {
    uint8_t* za = b3 + 64 * 64 * 2;
    const __nv_bfloat16 hi = __float2bfloat16_rn(zv);
    const float r1 = zv - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    *reinterpret_cast<__nv_bfloat16*>(za + sw128_off(dk, 0)) = hi;
    *reinterpret_cast<__nv_bfloat16*>(za + sw128_off(dk, 1)) = mid;
    *reinterpret_cast<__nv_bfloat16*>(za + sw128_off(dk, 2)) = lo;
}

// The three split products D (+)= A * B over K = 64 in steps of 16: hi*hi,
// hi*lo, lo*hi. a(kk, part) / b(kk, part) give the descriptors of step kk of
// the hi (part 0) or lo (part 1) operand; the first product overwrites D
// unless `acc`.
template <typename FA, typename FB>
__device__ __forceinline__ void mma_split(uint32_t d, FA a, FB b, uint32_t idesc, bool acc) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        mma_bf16(d, a(kk, 0), b(kk, 0), idesc, (acc || kk > 0) ? 1u : 0u);
        mma_bf16(d, a(kk, 0), b(kk, 1), idesc, 1u);
        mma_bf16(d, a(kk, 1), b(kk, 0), idesc, 1u);
    }
}

template <int MODE, int PHI>
__global__ void __launch_bounds__(F32Cfg<MODE>::THREADS, F32Cfg<MODE>::MIN_BLOCKS)
tc_f32_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
              const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mOut,
              const float* __restrict__ state_in, const float* __restrict__ z_in, float* __restrict__ rec_out,
              int H, int N, int block_tokens, int nblk, int group, const int32_t* __restrict__ perm,
              const int32_t* __restrict__ bin_start, const int32_t* __restrict__ msort, int nbins, int normalize,
              float* __restrict__ out, uint32_t* __restrict__ err) {
    using CF = F32Cfg<MODE>;
    constexpr int D = CF::D, C = CF::C;
    constexpr bool mapped = PHI != PHI_IDENTITY;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* stages = align1024(smem_raw);
    uint8_t* pt = stages + CF::STAGES * CF::STAGE;
    uint8_t* b3 = pt + 2 * CF::PT;
    uint8_t* qg = b3 + CF::NB3 * CF::B3;
    uint8_t* stg = qg + CF::QG;
    int* rows = reinterpret_cast<int*>(stg + CF::STG);  // [query slot][token C | key limit C]
    float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(rows) + CF::ROWS);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + CF::RED);
    uint64_t* empty = full + CF::STAGES;
    // Per stage: the chunk's tiles split (and the state operands written). In
    // kState and kReadout the prep warps may run up to STAGES chunks ahead of
    // the MMA warp; they reach barrier s again only after the MMA warp has
    // released stage s, so no barrier completes a second phase before its
    // waiter has seen the first (which a parity wait could not tell apart).
    uint64_t* bprep = empty + CF::STAGES;
    uint64_t* bsdone = bprep + CF::STAGES;  // S update of the chunk (kState: of the block) done
    uint64_t* bpfull = bsdone + 1;         // [2] P ready
    uint64_t* bptready = bpfull + 2;       // [2] P~ written (P read)
    uint64_t* bofull = bptready + 2;       // [2] O, Oz ready
    uint64_t* bofree = bofull + 2;         // [2] O, Oz read
    // gathered query tiles, per query slot (tile t uses t % QS, phase t / QS):
    // rows landed with their row table, queries split, slot read out
    uint64_t* qfull = bofree + 2;
    uint64_t* bqready = qfull + CF::QS;
    uint64_t* qfree = bqready + CF::QS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfree + CF::QS);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // CTA x takes `group` consecutive blocks of block_tokens (kSweep: the
    // sweep carries the state from one to the next, so it seeds from the
    // first block's record); records are indexed with the plan's nblk
    const int blk = blockIdx.x * group;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int nchunks = (N + C - 1) / C;
    const int c_begin = blk * (block_tokens / C);
    // the prefix mask's last block also answers the bin past the last chunk
    // (queries with m_i = N - 1 when C divides N)
    const int c_end = (CF::GATHER && blk == nblk - 1) ? nbins : min(nchunks, c_begin + group * (block_tokens / C));
    const int nci = c_end - c_begin;
    constexpr size_t kRec = (size_t)D * D + D;
    const size_t hoff = (size_t)bh * N * D;
    // query tiles answered at chunk c: one (its own queries) or the bin's
    auto q_tiles = [&](int c) -> int {
        if (!CF::GATHER) return CF::OUT ? 1 : 0;
        const int cnt = bin_start[(size_t)b * (nbins + 1) + c + 1] - bin_start[(size_t)b * (nbins + 1) + c];
        return (cnt + C - 1) / C;
    };

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int s = 0; s < CF::STAGES; ++s) mbar_init(bprep + s, 128);
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
        if (CF::OUT) tma_prefetch_map(&mQ);
        if (CF::OUT && !CF::GATHER) tma_prefetch_map(&mOut);
        if (CF::HAS_KV) {
            tma_prefetch_map(&mK);
            tma_prefetch_map(&mV);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // kState is the first kernel of its call: nothing is read before the
    // previous kernel on the stream is done. The later kernels let the TMA
    // warp load the caller's inputs first; every other warp waits before it
    // reads what the call's earlier kernels wrote.
    if (MODE == kState || warp != 0) pdl_wait();

    if (warp == 0) {
        // ---------------- TMA producer (whole warp) ----------------
        auto load_chunk = [&](int ci) {
            const int s = ci % CF::STAGES;
            if (lane == 0) {
                mbar_arrive_expect_tx(full + s, CF::STAGE);
                uint8_t* st = stages + s * CF::STAGE;
                const int row = (c_begin + ci) * C;
#pragma unroll
                for (int bx = 0; bx < 2; ++bx) {
                    if (CF::HAS_Q) tma_load_3d(st + bx * 8192, &mQ, full + s, bx * 32, row, bh);
                    if (CF::HAS_KV) {
                        tma_load_3d(st + CF::OFF_K + bx * 8192, &mK, full + s, bx * 32, row, bh);
                        tma_load_3d(st + CF::OFF_V + bx * 8192, &mV, full + s, bx * 32, row, bh);
                    }
                }
            }
        };
        int nld = min(nci, CF::STAGES);
        for (int ci = 0; ci < nld; ++ci) load_chunk(ci);
        // the bin tables below come from an earlier kernel of the call
        if (CF::GATHER) pdl_wait();
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
            if (CF::GATHER) {
                // the chunk's query tiles: rows of bin c, key limits relative to the chunk
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
                    if (lane == 0) mbar_arrive_expect_tx(qfull + slot, CF::FT);
                    __syncwarp();
                    gather_tile<C, 2, 32>(qg + slot * CF::FT, &mQ, qfull + slot, bh * N, tok, lane);
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
            constexpr uint32_t idS = idesc_bf16(D, D, true, true);    // S += K^T V
            constexpr uint32_t idP = idesc_bf16(C, C, false, false);  // P = Q K^T
            constexpr uint32_t idO = idesc_bf16(C, D, false, true);   // O += P~ V ; O += Q S_lo
            constexpr uint32_t idOZ = idesc_bf16(C, D + 16, false, true);  // O = Q [S_hi | z parts]
            constexpr uint32_t LO = CF::LO;
            const uint32_t pta = smem_u32(pt);
            bool ok = true;
            int tq = 0;
            for (int ci = 0; ci < nci && ok; ++ci) {
                const int s = ci % CF::STAGES;
                const uint32_t st = smem_u32(stages + s * CF::STAGE);
                const uint32_t kt = st + CF::OFF_K, vt = st + CF::OFF_V;
                ok = mbar_wait(bprep + s, (ci / CF::STAGES) & 1, err);
                if (!ok) break;
                tc_fence_after();
                // operand descriptors (part 0: hi tile, part 1: lo tile)
                auto kT = [&](int kk, int part) { return sdesc(kt + part * LO + kk * 2048, C * 128, 1024); };
                auto vN = [&](int kk, int part) { return sdesc(vt + part * LO + kk * 2048, C * 128, 1024); };
                auto kK = [&](int kk, int part) { return sdesc(kt + part * LO + kk * 32, 16, 1024); };
                if (MODE != kReadout) {
                    mma_split(tmem + CF::COL_S, kT, vN, idS, CF::SWEEP || ci > 0);
                    if (CF::SWEEP) mma_commit(bsdone);
                }
                const uint32_t b3a = smem_u32(b3 + (CF::SWEEP ? (ci & 1) * CF::B3 : 0));
                const int ntq = q_tiles(c_begin + ci);
                for (int t = 0; t < ntq && ok; ++t, ++tq) {
                    const int j = tq & 1, k = tq >> 1;  // accumulator slot of the tile, use of the slot
                    const int qs = tq % CF::QS;         // query slot (gathered tiles)
                    const uint32_t qt = CF::GATHER ? smem_u32(qg + qs * CF::FT) : st;
                    auto qK = [&](int kk, int part) { return sdesc(qt + part * LO + kk * 32, 16, 1024); };
                    if (CF::GATHER) ok = mbar_wait(bqready + qs, (tq / CF::QS) & 1, err);
                    if (CF::SWEEP) {
                        if (ok && k > 0) ok = mbar_wait(bptready + j, (k - 1) & 1, err);  // P[j] read two tiles ago
                        if (!ok) break;
                        tc_fence_after();
                        mma_split(tmem + CF::COL_P + slot_lanes(j), qK, kK, idP, false);
                        mma_commit(bpfull + j);
                    }
                    if (ok && k > 0) ok = mbar_wait(bofree + j, (k - 1) & 1, err);  // O[j] read two tiles ago
                    if (!ok) break;
                    tc_fence_after();
                    // O (80 columns) = Q_hi [S_hi | z] + Q_hi S_lo + Q_lo [S_hi | z]; the
                    // hi operand spans two swizzle atoms along N (stride one atom)
                    const uint32_t od = tmem + CF::COL_O + slot_lanes(j);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t shz = sdesc(b3a + kk * 2048, CF::ATOM, 1024);
                        const uint64_t slo = sdesc(b3a + 2 * CF::ATOM + kk * 2048, CF::ATOM, 1024);
                        mma_bf16(od, qK(kk, 0), shz, idOZ, kk > 0 ? 1u : 0u);
                        mma_bf16(od, qK(kk, 0), slo, idO, 1u);
                        mma_bf16(od, qK(kk, 1), shz, idOZ, 1u);
                    }
                    if (CF::SWEEP) {
                        ok = mbar_wait(bptready + j, k & 1, err);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t ptj = pta + j * CF::PT;
                        auto pK = [&](int kk, int part) { return sdesc(ptj + part * (C * C * 2) + kk * 32, 16, 1024); };
                        mma_split(tmem + CF::COL_O + slot_lanes(j), pK, vN, idO, true);
                    }
                    mma_commit(bofull + j);
                }
                mma_commit(empty + s);
            }
            if (MODE == kState) mma_commit(bsdone);  // the block's state is complete
        }
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        // the z atoms start zero (columns 3..15 stay so; unnormalized, all)
        for (int x = et; x < CF::NB3 * CF::ATOM / 16; x += 128) {
            const int buf = x / (CF::ATOM / 16), q = x % (CF::ATOM / 16);
            reinterpret_cast<uint4*>(b3 + buf * CF::B3 + CF::ATOM)[q] = make_uint4(0, 0, 0, 0);
        }
        float zp = 0.f;  // z entry d_k = et (threads et < 64) of the running state
        if (CF::SWEEP) {
            // seed S (TMEM, M = 64: row a in lane a % 16 of sub-partition a / 16)
            // and z from the block's prefix record
            const float* pre = state_in + ((size_t)bh * nblk + blk) * kRec;
            const int a = sp * 16 + (lane & 15);
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
            tmem_st_wait();
            if (et < D) zp = pre[(size_t)D * D + et];
        } else if (MODE == kReadout) {
            // the head's total state, split once
            const float* S = state_in + (size_t)bh * D * D;
            const int a = et >> 1, c0 = (et & 1) * 32;
            float f[32];
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
                const float4 x = reinterpret_cast<const float4*>(S + (size_t)a * D + c0)[q4];
                f[4 * q4] = x.x;
                f[4 * q4 + 1] = x.y;
                f[4 * q4 + 2] = x.z;
                f[4 * q4 + 3] = x.w;
            }
            split_state_row(b3, a, c0, f);
            if (normalize && et < D) split_z(b3, et, z_in[(size_t)bh * D + et]);
        }
        int tq = 0;
        for (int ci = 0; ci < nci; ++ci) {
            const int c = c_begin + ci;
            const int s = ci % CF::STAGES, u = ci / CF::STAGES;
            const int valid = c < nchunks ? min(C, N - c * C) : 0;
            uint8_t* st = stages + s * CF::STAGE;
            mbar_wait(full + s, u & 1, err);
            if (CF::HAS_Q) split_tile<PHI, mapped>(st, et, C, nullptr);
            if (CF::HAS_KV) {
                float cs[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) cs[e] = 0.f;
                split_tile<PHI, mapped>(st + CF::OFF_K, et, valid, cs);
                // lanes l, l ^ 8, l ^ 16, l ^ 24 hold the same column group
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 8);
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 16);
                }
                float* rp = red + (ci & 1) * 4 * D;
                if (lane < 8) {
                    float4* dst = reinterpret_cast<float4*>(rp + (warp - 2) * D + 8 * lane);
                    dst[0] = make_float4(cs[0], cs[1], cs[2], cs[3]);
                    dst[1] = make_float4(cs[4], cs[5], cs[6], cs[7]);
                }
                // the V tile's barrier also publishes the partials above
                split_tile<PHI, false>(st + CF::OFF_V, et, C, nullptr);
            }
            if (CF::SWEEP) {
                if (ci > 0) {
                    mbar_wait(bsdone, (ci - 1) & 1, err);
                    tc_fence_after();
                }
                // S_prev -> hi / lo operands (row d_k = a, columns cb .. cb + 31)
                const int a = sp * 16 + (lane & 15);
                const int cb = lane < 16 ? 0 : 32;
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + CF::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + CF::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
                float f[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(r[e]);
                split_state_row(b3 + (ci & 1) * CF::B3, a, cb, f);
                if (normalize && et < D) split_z(b3 + (ci & 1) * CF::B3, et, zp);
            }
            if (CF::HAS_KV && et < D) {
                const float* rp = red + (ci & 1) * 4 * D;
                zp += (rp[et] + rp[D + et]) + (rp[2 * D + et] + rp[3 * D + et]);
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep + s);
            if (CF::GATHER) {
                // the gathered query rows of the chunk's tiles: phi and the split in place
                const int ntq = q_tiles(c);
                for (int t = 0; t < ntq; ++t, ++tq) {
                    const int slot = tq % CF::QS;
                    mbar_wait(qfull + slot, (tq / CF::QS) & 1, err);
                    split_tile<PHI, mapped>(qg + slot * CF::FT, et, C, nullptr);
                    fence_async_smem();
                    mbar_arrive(bqready + slot);
                }
            }
        }
        if (MODE == kState && et < D) rec_out[((size_t)bh * nblk + blk) * kRec + (size_t)D * D + et] = zp;
    } else {
        // ---------------- mask + epilogue warps ----------------
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int i = sp * 16 + (lane & 15);  // accumulator row (query, or d_k in kState)
        const int half = lane >= 16 ? 1 : 0;  // the two warp halves take the two column halves
        if (MODE == kState) {
            // the block's S: row d_k = i, columns 32 half .. 32 half + 31
            const bool ok = mbar_wait(bsdone, 0, err);
            tc_fence_after();
            uint32_t r[32];
            tmem_ld16x2<32>(tmem + CF::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
            tmem_ld16x2<32>(tmem + CF::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
            tmem_ld_wait();
            if (ok) {
                float4* dst = reinterpret_cast<float4*>(rec_out + ((size_t)bh * nblk + blk) * kRec + (size_t)i * D +
                                                        32 * half);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4)
                    dst[q4] = make_float4(__uint_as_float(r[4 * q4]), __uint_as_float(r[4 * q4 + 1]),
                                          __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3]));
            }
        } else {
            // No early exit in this warpgroup (named barrier 3); a failed wait
            // only suppresses the output stores.
            bool ok = true;
            const int et2 = threadIdx.x - 192;
            int tq = 0;
            for (int ci = 0; ci < nci; ++ci) {
                const int c = c_begin + ci;
                const int ntq = q_tiles(c);
                for (int t = 0; t < ntq; ++t, ++tq) {
                    const int slot = tq & 1, use = tq >> 1;
                    const int qs = tq % CF::QS;
                    const uint32_t lane_s = lane_base + slot_lanes(slot);
                    float rs = 0.f;
                    int dst = -1;  // gathered: the token of output row i
                    if (CF::SWEEP) {
                        ok = mbar_wait(bpfull + slot, use & 1, err) && ok;
                        // the row table of a gathered tile (written by the TMA warp)
                        if (CF::GATHER) ok = mbar_wait(qfull + qs, (tq / CF::QS) & 1, err) && ok;
                        tc_fence_after();
                        const int* srow = rows + qs * 2 * C;
                        const int lim = CF::GATHER ? srow[C + i] : i;  // last key of the chunk row i sees
                        if (CF::GATHER) dst = srow[i];
                        uint32_t r[32];
                        tmem_ld16x2<32>(tmem + CF::COL_P + lane_s, *reinterpret_cast<uint32_t(*)[16]>(r));
                        tmem_ld16x2<32>(tmem + CF::COL_P + lane_s + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                        tmem_ld_wait();
                        uint8_t* pts = pt + slot * CF::PT;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const int jk = 32 * half + 8 * g + e;  // key within the chunk
                                f[e] = jk <= lim ? __uint_as_float(r[8 * g + e]) : 0.f;
                                rs += f[e];
                            }
                            uint4 hi, lo;
                            split8(f, hi, lo);
                            *reinterpret_cast<uint4*>(pts + sw128_off(i, 32 * half + 8 * g)) = hi;
                            *reinterpret_cast<uint4*>(pts + C * C * 2 + sw128_off(i, 32 * half + 8 * g)) = lo;
                        }
                        rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                        fence_async_smem();
                        tc_fence_before();
                        mbar_arrive(bptready + slot);
                    }
                    // epilogue: this thread's half of output row i
                    ok = ok && mbar_wait(bofull + slot, use & 1, err);
                    tc_fence_after();
                    uint32_t o[32];
                    tmem_ld16x2<32>(tmem + CF::COL_O + lane_s, *reinterpret_cast<uint32_t(*)[16]>(o));
                    tmem_ld16x2<32>(tmem + CF::COL_O + lane_s + 16, *reinterpret_cast<uint32_t(*)[16]>(o + 16));
                    // Oz: a 32x32b load starts at the sub-partition's lane 0, so
                    // slot 1 (lanes 16..31) is picked out below with a shuffle
                    uint32_t oz[4];
                    tmem_ld4(tmem + CF::COL_OZ + lane_base, oz);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(bofree + slot);
                    if (CF::GATHER) mbar_arrive(qfree + qs);  // the query slot and its row table are read
                    float den = rs + (__uint_as_float(oz[0]) + __uint_as_float(oz[1]) + __uint_as_float(oz[2]));
                    den = __shfl_sync(0xffffffffu, den, (lane & 15) + 16 * slot);
                    const float inv = normalize ? 1.0f / den : 1.0f;
                    if (CF::GATHER) {
                        // gathered rows go out directly: 128 bytes of row dst per thread
                        if (ok && dst >= 0) {
                            float4* op = reinterpret_cast<float4*>(out + hoff + (size_t)dst * D + 32 * half);
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4)
                                op[q4] = make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                                     __uint_as_float(o[4 * q4 + 2]) * inv,
                                                     __uint_as_float(o[4 * q4 + 3]) * inv);
                        }
                    } else {
                        if (et2 == 0) bulk_wait_read0();  // the previous tile's store has read the staging tile
                        named_bar(3, 128);
                        uint8_t* row = stg + half * 8192 + i * 128;
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            *reinterpret_cast<float4*>(row + ((q4 ^ (i & 7)) << 4)) =
                                make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                            __uint_as_float(o[4 * q4 + 2]) * inv, __uint_as_float(o[4 * q4 + 3]) * inv);
                        fence_async_smem();
                        named_bar(3, 128);
                        if (et2 == 0 && ok) {
                            tma_store_3d(&mOut, stg, 0, c * C, bh);
                            tma_store_3d(&mOut, stg + 8192, 32, c * C, bh);
                            bulk_commit();
                        }
                    }
                }
            }
        }
    }
    if (CF::OUT && !CF::GATHER && threadIdx.x == 192) bulk_wait0();  // the output stores have landed
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, CF::TMEM_COLS);
    }
}

// fp32 [bh][N][64] tensor, boxes of 32 columns x 64 rows, 128-byte swizzle
cudaError_t make_map_f32(CUtensorMap* map, const void* base, int N, long long bh) {
    return make_map_box(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 64, N, bh, 32, 64);
}

struct F32Args {
    const void *q, *k, *v;
    const float *state_in, *z_in;
    float* rec_out;
    int block_tokens, nblk;
    const int32_t *perm, *bins, *msort;
    int nbins;
    void* out;
};

template <int MODE, int PHI>
cudaError_t launch_f32(const Problem& p, const F32Args& a, uint32_t* err, cudaStream_t st) {
    using CF = F32Cfg<MODE>;
    if (p.d != CF::D || p.dtype != DT_F32 || a.block_tokens % CF::C != 0) return cudaErrorInvalidValue;
    CUtensorMap mq{}, mk{}, mv{}, mo{};
    cudaError_t e = cudaSuccess;
    if (CF::GATHER) {
        // gathered query rows: a 2-D row map for tile::gather4 (boxes of 32 fp32 columns x 1 row)
        e = make_row_map_box(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 64, p.bh() * p.N, 32);
    } else if (CF::HAS_Q) {
        e = make_map_f32(&mq, a.q, p.N, p.bh());
        if (e == cudaSuccess) e = make_map_f32(&mo, a.out, p.N, p.bh());
    }
    if (e == cudaSuccess && CF::HAS_KV) {
        e = make_map_f32(&mk, a.k, p.N, p.bh());
        if (e == cudaSuccess) e = make_map_f32(&mv, a.v, p.N, p.bh());
    }
    if (e != cudaSuccess) return e;
    e = ensure_smem<tc_f32_kernel<MODE, PHI>>(CF::SMEM);
    if (e != cudaSuccess) return e;
    // the causal sweep holds one CTA per SM: it takes several blocks per CTA
    // when the plan has more (block, head) pairs than SMs, so that one wave
    // runs (the prefix mask keeps one block per CTA: its last block answers
    // the bins past the plan's chunks)
    int group = 1;
    if (MODE == kSweep) {
        const long long pairs = (long long)a.nblk * p.bh();
        group = (int)std::min<long long>(a.nblk, (pairs + device_sms() - 1) / device_sms());
    }
    dim3 grid((a.nblk + group - 1) / group, (unsigned)p.bh());
    return launch_pdl(tc_f32_kernel<MODE, PHI>, grid, dim3(CF::THREADS), CF::SMEM, st, mq, mk, mv, mo, a.state_in,
                      a.z_in, a.rec_out, p.H, p.N, a.block_tokens, a.nblk, group, a.perm, a.bins, a.msort, a.nbins,
                      p.normalize, static_cast<float*>(a.out), err);
}

template <int MODE>
cudaError_t launch_phi(const Problem& p, const F32Args& a, uint32_t* err, cudaStream_t st) {
    switch (p.phi) {
        case PHI_RELU1:
            return launch_f32<MODE, PHI_RELU1>(p, a, err, st);
        case PHI_ELU1:
            return launch_f32<MODE, PHI_ELU1>(p, a, err, st);
        default:
            return launch_f32<MODE, PHI_IDENTITY>(p, a, err, st);
    }
}

}  // namespace

bool tc_f32_supported(const Problem& p) { return p.dtype == DT_F32 && p.d == 64; }

cudaError_t tc_f32_states(const Problem& p, const void* k, const void* v, int block_tokens, int nblk, float* part,
                          uint32_t* err, cudaStream_t st) {
    const F32Args a{nullptr, k, v, nullptr, nullptr, part, block_tokens, nblk, nullptr, nullptr, nullptr, 0, nullptr};
    return launch_phi<kState>(p, a, err, st);
}

cudaError_t tc_f32_chunked(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                           int block_tokens, int nblk, void* out, uint32_t* err, cudaStream_t st) {
    const F32Args a{q, k, v, prefix, nullptr, nullptr, block_tokens, nblk, nullptr, nullptr, nullptr, 0, out};
    return launch_phi<kSweep>(p, a, err, st);
}

cudaError_t tc_f32_prefix(const Problem& p, const void* q, const void* k, const void* v, const float* prefix,
                          int block_tokens, int nblk, const int32_t* perm, const int32_t* bins, const int32_t* msort,
                          int nbins, void* out, uint32_t* err, cudaStream_t st) {
    const F32Args a{q, k, v, prefix, nullptr, nullptr, block_tokens, nblk, perm, bins, msort, nbins, out};
    return launch_phi<kGather>(p, a, err, st);
}

cudaError_t tc_f32_readout(const Problem& p, const void* q, const float* S, const float* z, int block_tokens,
                           int nblk, void* out, uint32_t* err, cudaStream_t st) {
    const F32Args a{q, nullptr, nullptr, S, z, nullptr, block_tokens, nblk, nullptr, nullptr, nullptr, 0, out};
    return launch_phi<kReadout>(p, a, err, st);
}

}  // namespace la
