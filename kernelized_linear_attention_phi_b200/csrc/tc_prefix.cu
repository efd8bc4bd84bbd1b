// Prefix-mask attention in one kernel for sequences of at most 4096 tokens
// (bf16, d = 64) on tcgen05 tensor cores.
//
// The form ("trim-transformer 0.1.0", "Masking"): query i of a sequence sees
// keys 0..m_i; out_i = sum_{j <= m_i} (phi(q_i).phi(k_j)) v_j, divided by
// sum_{j <= m_i} phi(q_i).phi(k_j) when normalized.
//
// Each head is cut into NC blocks of BT keys (a multiple of 128), one CTA per
// block, the NC CTAs of a head forming one thread-block cluster. CTA r
// answers every query whose key limit m_i lies in its block [r*BT, r*BT+BT):
//
//   phase A  the block's state T_r = phi(K_r)^T V_r, z_r = phi(K_r)^T 1
//            (tensor cores, over the block's 128-key sub-blocks; for relu+1
//            as relu(K)^T V + 1 (x) colsum(V) and colsum(relu K) + count,
//            relu(K) being exact in bf16, so the state carries no rounding of
//            phi(K)); meanwhile
//            the mask warps bin the sequence's queries: those with m_i in
//            the block, stably sorted by the sub-block holding m_i;
//   phase B  the block prefix S_bp = sum_{r' < r} T_r' (and z) over
//            distributed shared memory after a cluster barrier;
//   phase D  a sweep over the block's sub-blocks k = 0..nsub-1 with the
//            running state S_k = S_bp + sum_{k' < k} T_k' in TMEM. The sorted
//            queries are cut into tiles of 128 in order; a tile whose first
//            query's limit lies in sub-block k starts there with
//            O = phi(Q) S_k (and phi(Q).z_k for the denominator), then takes
//            at every sub-block kk from k to the sub-block of its last query
//            P = phi(Q) phi(K_kk)^T, P~ = P with keys j > m_i zeroed (bf16;
//            row sums kept in fp32), O += P~ V_kk. So each query sees the
//            state of every key before its tile's first sub-block plus its
//            own keys from there to m_i. Tiles are contiguous in the sorted
//            order, so at most one tile stays open from one sub-block to the
//            next.
//
// Warp roles (320 threads): warp 0 TMA (K / V sub-blocks through a two-stage
// ring, twice: phase A and phase D; query tiles gathered by tile::gather4
// through a 2-D row map of Q), warp 1 TMEM owner and MMA issuer, warps 2-5
// "prep" (phi on the K and Q tiles, the state exchange, S_k -> bf16
// operands), warps 6-9 "mask" (binning in phase A, then P~ and the
// epilogues). One CTA per SM (shared memory), TMEM: S, z, two P slots, two
// O slots.

#include <algorithm>

#include "device.h"
#include "launch_util.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

using namespace tc;

struct PfCfg {
    static constexpr int D = 64;
    static constexpr int KC = 128;                     // keys per sub-block = queries per tile
    static constexpr int NMAX = 4096;                  // longest sequence
    static constexpr int MAX_SUB = NMAX / KC;          // sub-blocks per block at most
    static constexpr int MAX_TILES = NMAX / KC;        // query tiles per block at most
    static constexpr int MAX_OPS = MAX_TILES + MAX_SUB;
    static constexpr int LIM_BITS = 13;                // table entry: token << 13 | limit in block
    static constexpr int TILE = KC * D * 2;            // one [128 x 64] bf16 tile
    static constexpr int STAGES = 2;                   // K / V ring
    static constexpr int STAGE = 2 * TILE;             // K, V
    static constexpr int QB = 2;                       // query tile buffers
    static constexpr int PT = KC * KC * 2;             // P~ [128 x 128] bf16: two 64-key boxes
    static constexpr int B3 = D * D * 2;               // S_k, bf16, MN-major
    static constexpr int BZ = 16 * D * 2;              // [z_hi; z_lo; 0], K-major
    static constexpr int ONES = 16 * KC * 2;           // all-ones [16 x 128], K-major, two boxes
    static constexpr int XCH = (D * D + D) * 4;        // the block's state, fp32 (read by the cluster)
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_Q = OFF_RING + STAGES * STAGE;
    static constexpr int OFF_PT = OFF_Q + QB * TILE;
    static constexpr int OFF_B3 = OFF_PT + 2 * PT;
    static constexpr int OFF_BZ = OFF_B3 + 2 * B3;
    static constexpr int OFF_ONES = OFF_BZ + 2 * BZ;
    static constexpr int OFF_XCH = OFF_ONES + ONES;
    static constexpr int OFF_TAB = OFF_XCH + XCH;
    static constexpr int OFF_OPS = OFF_TAB + NMAX * 4;
    static constexpr int OFF_STEP = OFF_OPS + MAX_OPS * 4;
    static constexpr int OFF_BIN = OFF_STEP + (MAX_SUB + 1) * 4;     // hist, base per mask warp and bucket
    static constexpr int OFF_MISC = OFF_BIN + 2 * 4 * MAX_SUB * 4;  // nq, nt, nops, tmem base
    static constexpr int NBAR = 2 * STAGES + STAGES + 3 + 4 * 2 + 3 * QB;
    static constexpr int OFF_BAR = (OFF_MISC + 64 + 15) / 16 * 16;  // mbarriers are 8-byte aligned
    static constexpr size_t SMEM = 1024 + (size_t)OFF_BAR + 8 * NBAR;
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(OFF_Q % 1024 == 0 && OFF_PT % 1024 == 0 && OFF_B3 % 1024 == 0 && OFF_BZ % 1024 == 0 &&
                      OFF_ONES % 1024 == 0,
                  "128-byte-swizzled tiles start on 1024-byte boundaries");
    static_assert(XCH <= PT, "the block prefix is staged in the first P~ buffer");
    static_assert(NMAX * 4 <= PT, "the mask row is staged in the second P~ buffer");
    static_assert(OFF_XCH % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
    // TMEM columns: S (M = 64) and z, two P slots (M = 128, N = 128), two O
    // slots (O, then Oz)
    static constexpr int COL_S = 0, COL_Z = D, COL_P = D + 16, COL_O = COL_P + 2 * KC, OSLOT = D + 16;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_O + 2 * OSLOT <= (int)TMEM_COLS, "TMEM");
    static constexpr int THREADS = 320;
};

// An op of phase D: tile t at sub-block k, and whether it opens / closes the tile.
__device__ __forceinline__ int op_pack(int t, int k, bool opens, bool closes) {
    return (t << 16) | (k << 8) | (opens ? 1 : 0) | (closes ? 2 : 0);
}
__device__ __forceinline__ int op_tile(int op) { return op >> 16; }
__device__ __forceinline__ int op_sub(int op) { return (op >> 8) & 0xFF; }
__device__ __forceinline__ bool op_opens(int op) { return op & 1; }
__device__ __forceinline__ bool op_closes(int op) { return op & 2; }

// CAUSAL: the causal form (m_i = i) without a mask: the queries of the block
// are its own tokens, so no binning; tile t is sub-block t (loaded as a TMA
// tile, not gathered) and has exactly one op.
template <int PHI, bool CAUSAL>
__global__ void __launch_bounds__(PfCfg::THREADS, 1)
tc_prefix_fused_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                       const __grid_constant__ CUtensorMap mV, const int32_t* __restrict__ m, int H, int N,
                       int block_tokens, int normalize, __nv_bfloat16* __restrict__ out, float* __restrict__ S_total,
                       float* __restrict__ z_total, uint32_t* __restrict__ err) {
    using CF = PfCfg;
    constexpr int D = CF::D, KC = CF::KC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = align1024(smem_raw);
    uint8_t* ring = base + CF::OFF_RING;
    uint8_t* qbuf = base + CF::OFF_Q;
    uint8_t* pt = base + CF::OFF_PT;
    uint8_t* b3 = base + CF::OFF_B3;
    uint8_t* bz = base + CF::OFF_BZ;
    uint8_t* ones = base + CF::OFF_ONES;
    float* xch = reinterpret_cast<float*>(base + CF::OFF_XCH);
    int* tab = reinterpret_cast<int*>(base + CF::OFF_TAB);
    int* ops = reinterpret_cast<int*>(base + CF::OFF_OPS);
    int* step_begin = reinterpret_cast<int*>(base + CF::OFF_STEP);
    int* hist = reinterpret_cast<int*>(base + CF::OFF_BIN);         // [4][MAX_SUB]
    int* bbase = hist + 4 * CF::MAX_SUB;                            // [4][MAX_SUB]
    int* misc = reinterpret_cast<int*>(base + CF::OFF_MISC);        // nq, nt, nops, tmem
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + CF::OFF_BAR);
    uint64_t* full = bars;                       // [STAGES] K / V landed
    uint64_t* empty = full + CF::STAGES;         // [STAGES] K / V read by the MMAs
    uint64_t* kready = empty + CF::STAGES;       // [STAGES] K transformed (prep)
    uint64_t* bprep = kready + CF::STAGES;       // S_k operands ready (prep), once per sub-block of phase D
    uint64_t* bsdone = bprep + 1;                // state MMAs complete: end of phase A, then each sub-block
    uint64_t* binned = bsdone + 1;               // queries binned, op list written (mask)
    uint64_t* pfull = binned + 1;                // [2] P ready
    uint64_t* ptready = pfull + 2;               // [2] P~ written, P read (mask)
    uint64_t* ofull = ptready + 2;               // [2] O of a tile final
    uint64_t* ofree = ofull + 2;                 // [2] O read out (mask)
    uint64_t* qfull = ofree + 2;                 // [QB] query tile landed
    uint64_t* qready = qfull + CF::QB;           // [QB] query tile transformed (prep)
    uint64_t* qempty = qready + CF::QB;          // [QB] query tile read by the MMAs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 3);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int rank = blockIdx.x;  // cluster rank = block of the head
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int k0 = rank * block_tokens;
    const int nkeys = max(0, min(block_tokens, N - k0));
    const int nsub = (nkeys + KC - 1) / KC;  // the block's sub-blocks (every block has keys)
    constexpr bool mapped = PHI != PHI_IDENTITY;

    if (threadIdx.x == 0) {
        cta_abort_reset();
        for (int s = 0; s < CF::STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
            mbar_init(kready + s, 128);
        }
        mbar_init(bprep, 128);
        mbar_init(bsdone, 1);
        mbar_init(binned, 1);
        for (int j = 0; j < 2; ++j) {
            mbar_init(pfull + j, 1);
            mbar_init(ptready + j, 128);
            mbar_init(ofull + j, 1);
            mbar_init(ofree + j, 128);
        }
        for (int j = 0; j < CF::QB; ++j) {
            mbar_init(qfull + j, 1);
            mbar_init(qready + j, 128);
            mbar_init(qempty + j, 1);
        }
        fence_mbar_init();
        tma_prefetch_map(&mQ);
        tma_prefetch_map(&mK);
        tma_prefetch_map(&mV);
    }
    if (warp == 1) tmem_alloc(tmem_slot, CF::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The only kernel of its call: the kernel before it on the stream may have
    // written this call's inputs, so every warp waits for it first.
    pdl_wait();

    // Phase-B cluster barrier: every thread arrives once (after the work of
    // phase A it must not hold up) and waits once; the prep warps wait at
    // once, the others only before the final barrier.
    bool phase_b_waited = false;

    if (warp == 0) {
        // ---------------- TMA producer (whole warp) ----------------
        bool ok = true;
        int nld = 0;  // loads issued: phase A sub-blocks 0..nsub-1, then phase D again
        auto load = [&](int ld) {
            const int s = ld % CF::STAGES, u = ld / CF::STAGES;
            if (ld >= CF::STAGES) ok = ok && __all_sync(0xffffffffu, mbar_wait(empty + s, (u - 1) & 1, err));
            if (!ok) return;
            if (lane == 0) {
                const int row = k0 + (ld % nsub) * KC;
                uint8_t* st = ring + s * CF::STAGE;
                mbar_arrive_expect_tx(full + s, CF::STAGE);
                tma_load_3d(st, &mK, full + s, 0, row, bh);
                tma_load_3d(st + CF::TILE, &mV, full + s, 0, row, bh);
            }
            nld = ld + 1;
        };
        for (int ld = 0; ld < nsub; ++ld) load(ld);
        asm volatile("barrier.cluster.arrive;" ::: "memory");
        ok = ok && __all_sync(0xffffffffu, mbar_wait(binned, 0, err));
        const int nq = misc[0];
        int tq = 0;  // query tiles issued
        for (int k = 0; k < nsub; ++k) {
            load(nsub + k);
            // the tiles that open at sub-block k
            for (int n = step_begin[k]; n < step_begin[k + 1]; ++n) {
                const int op = ops[n];
                if (!op_opens(op)) continue;
                const int t = op_tile(op), qb = t % CF::QB, u = t / CF::QB;
                if (t >= CF::QB) ok = ok && __all_sync(0xffffffffu, mbar_wait(qempty + qb, (u - 1) & 1, err));
                if (!ok) break;
                if (CAUSAL) {
                    // the block's own tokens (rows past N arrive as zeros)
                    if (lane == 0) {
                        mbar_arrive_expect_tx(qfull + qb, CF::TILE);
                        tma_load_3d(qbuf + qb * CF::TILE, &mQ, qfull + qb, 0, k0 + t * KC, bh);
                    }
                } else {
                    int tok[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int pos = t * KC + 4 * lane + e;
                        tok[e] = pos < nq ? (tab[pos] >> CF::LIM_BITS) : -1;
                    }
                    if (lane == 0) mbar_arrive_expect_tx(qfull + qb, CF::TILE);
                    __syncwarp();
                    gather_tile<KC, 1>(qbuf + qb * CF::TILE, &mQ, qfull + qb, bh * N, tok, lane);
                }
                tq = t + 1;
            }
        }
        // drain: the loads still in flight land before the CTA exits
        if (lane == 0) {
            for (int ld = max(0, nld - CF::STAGES); ld < nld; ++ld)
                mbar_wait(full + ld % CF::STAGES, (ld / CF::STAGES) & 1, err, false);
            for (int t = max(0, tq - CF::QB); t < tq; ++t) mbar_wait(qfull + t % CF::QB, (t / CF::QB) & 1, err, false);
        }
        (void)ok;
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // phase B needs nothing from this warp but its arrival
        asm volatile("barrier.cluster.arrive;" ::: "memory");
        if (lane == 0) {
            constexpr uint32_t id_su = idesc_bf16(D, D, true, true);     // S += K^T V
            constexpr uint32_t id_zu = idesc_bf16(D, 16, true, false);   // z += K^T 1
            constexpr uint32_t id_p = idesc_bf16(KC, KC, false, false);  // P = Q K^T
            constexpr uint32_t id_o = idesc_bf16(KC, D, false, true);    // O = Q S_k, O += P~ V
            constexpr uint32_t id_oz = idesc_bf16(KC, 16, false, false); // Oz = Q [z]
            constexpr uint32_t id_cs = idesc_bf16(D, D, false, true);    // 1 (x) colsum(V)
            const uint32_t onesa = smem_u32(ones), pta = smem_u32(pt), qa0 = smem_u32(qbuf);
            bool ok = true;
            // state MMAs over the sub-block in load `ld` (accumulating unless
            // `first`); with `colsum`, also colsum(V) into every row of the P
            // columns (an all-ones A operand; phase A of relu+1)
            auto state_update = [&](int ld, bool first, bool with_z, bool colsum) {
                const int s = ld % CF::STAGES;
                const uint32_t kt = smem_u32(ring + s * CF::STAGE), vt = kt + CF::TILE;
#pragma unroll
                for (int kk = 0; kk < KC / 16; ++kk) {
                    const uint64_t a = sdesc(kt + kk * 2048, KC * 128, 1024);
                    const uint64_t bv = sdesc(vt + kk * 2048, KC * 128, 1024);
                    const uint32_t acc = (first && kk == 0) ? 0u : 1u;
                    mma_bf16(tmem + CF::COL_S, a, bv, id_su, acc);
                    if (with_z)
                        mma_bf16(tmem + CF::COL_Z, a, sdesc(onesa + (kk / 4) * 2048 + (kk % 4) * 32, 16, 1024), id_zu,
                                 acc);
                    if (colsum)
                        mma_bf16(tmem + CF::COL_P, sdesc(pta + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024), bv,
                                 id_cs, acc);
                }
            };
            // phase A: the block's own state
            for (int ld = 0; ld < nsub && ok; ++ld) {
                const int s = ld % CF::STAGES;
                ok = mbar_wait(kready + s, (ld / CF::STAGES) & 1, err);
                if (!ok) break;
                tc_fence_after();
                state_update(ld, ld == 0, true, PHI == PHI_RELU1);
                mma_commit(empty + s);
            }
            mma_commit(bsdone);
            // phase D
            ok = ok && mbar_wait(binned, 0, err);
            const int nops = misc[2];
            int pending = -1;  // op whose P~ V is still to issue
            auto issue_pv = [&](int n) {
                const int op = ops[n], t = op_tile(op), k = op_sub(op), j = n & 1;
                const int ld = nsub + k, s = ld % CF::STAGES;
                ok = ok && mbar_wait(ptready + j, (n >> 1) & 1, err);
                if (!ok) return;
                tc_fence_after();
                const uint32_t vt = smem_u32(ring + s * CF::STAGE) + CF::TILE;
                const uint32_t ptj = pta + j * CF::PT;
                const uint32_t oc = tmem + CF::COL_O + (t & 1) * CF::OSLOT;
#pragma unroll
                for (int kk = 0; kk < KC / 16; ++kk)
                    mma_bf16(oc, sdesc(ptj + (kk / 4) * CF::TILE + (kk % 4) * 32, 16, 1024),
                             sdesc(vt + kk * 2048, KC * 128, 1024), id_o, 1u);
                if (op_closes(op)) {
                    mma_commit(ofull + (t & 1));
                    mma_commit(qempty + t % CF::QB);
                }
                if (n + 1 == nops || op_sub(ops[n + 1]) != k) mma_commit(empty + s);  // last op of sub-block k
            };
            for (int k = 0; k < nsub && ok; ++k) {
                const int ld = nsub + k, s = ld % CF::STAGES;
                // a P~ V deferred from sub-block k - 2 or earlier (sub-blocks
                // with no op in between) holds the ring slot this sub-block's
                // load is waiting for: issue it first
                if (pending >= 0 && op_sub(ops[pending]) + 2 <= k) {
                    issue_pv(pending);
                    pending = -1;
                    if (!ok) break;
                }
                ok = mbar_wait(bprep, k & 1, err) && mbar_wait(kready + s, (ld / CF::STAGES) & 1, err);
                if (!ok) break;
                tc_fence_after();
                state_update(ld, false, normalize != 0, false);
                mma_commit(bsdone);
                const uint32_t kt = smem_u32(ring + s * CF::STAGE);
                const uint32_t b3a = smem_u32(b3 + (k & 1) * CF::B3), bza = smem_u32(bz + (k & 1) * CF::BZ);
                const int n0 = step_begin[k], n1 = step_begin[k + 1];
                if (n0 == n1) mma_commit(empty + s);  // no tile touches this sub-block
                for (int n = n0; n < n1 && ok; ++n) {
                    const int op = ops[n], t = op_tile(op), j = n & 1;
                    const uint32_t qa = qa0 + (t % CF::QB) * CF::TILE;
                    const uint32_t oc = tmem + CF::COL_O + (t & 1) * CF::OSLOT;
                    if (op_opens(op)) {
                        ok = mbar_wait(qready + t % CF::QB, (t / CF::QB) & 1, err);
                        if (ok && t >= 2) ok = mbar_wait(ofree + (t & 1), ((t >> 1) - 1) & 1, err);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t a = sdesc(qa + kk * 32, 16, 1024);
                            mma_bf16(oc, a, sdesc(b3a + kk * 2048, D * 128, 1024), id_o, kk > 0);
                            if (normalize) mma_bf16(oc + D, a, sdesc(bza + kk * 32, 16, 1024), id_oz, kk > 0);
                        }
                    }
                    // P slot j was last read by the mask warps for op n - 2
                    if (n >= 2) ok = mbar_wait(ptready + j, ((n >> 1) - 1) & 1, err);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16(tmem + CF::COL_P + j * KC, sdesc(qa + kk * 32, 16, 1024), sdesc(kt + kk * 32, 16, 1024),
                                 id_p, kk > 0);
                    mma_commit(pfull + j);
                    if (pending >= 0) issue_pv(pending);
                    pending = n;
                }
            }
            if (ok && pending >= 0) issue_pv(pending);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------- prep warps ----------------
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const uint4 one8 = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        for (int c = et; c < CF::ONES / 16; c += 128) reinterpret_cast<uint4*>(ones)[c] = one8;
        for (int c = et; c < 2 * CF::BZ / 16; c += 128) reinterpret_cast<uint4*>(bz)[c] = make_uint4(0, 0, 0, 0);
        if (PHI == PHI_RELU1)  // phase A: an all-ones [64 x 128] A operand in the (idle) P~ buffers
            for (int c = et; c < 2 * D * 128 / 16; c += 128) reinterpret_cast<uint4*>(pt)[c] = one8;
        fence_async_smem();
        // phi on the K tile of load ld (phase A of relu+1: relu alone), rows
        // past the sequence zeroed
        auto transform_k = [&](int ld) {
            const int s = ld % CF::STAGES;
            mbar_wait(full + s, (ld / CF::STAGES) & 1, err);
            const int kvalid = min(KC, nkeys - (ld % nsub) * KC);
            if (mapped || kvalid < KC) {
                uint4* kt = reinterpret_cast<uint4*>(ring + s * CF::STAGE);
                constexpr int NL = CF::TILE / 16 / 128;
                const bool split = PHI == PHI_RELU1 && ld < nsub;
                uint4 w[NL];
#pragma unroll
                for (int j = 0; j < NL; ++j) w[j] = kt[et + 128 * j];
#pragma unroll
                for (int j = 0; j < NL; ++j) {
                    const int r = (et + 128 * j) >> 3;
                    kt[et + 128 * j] = r >= kvalid ? make_uint4(0, 0, 0, 0) : split ? relu_x8(w[j]) : phi8<PHI>(w[j]);
                }
                fence_async_smem();
            }
            mbar_arrive(kready + s);
        };
        // S (M = 64: rows in lanes 0..15 of each sub-partition) and z from TMEM
        const int a = sp * 16 + (lane & 15);  // d_k row of this thread
        const int cb = lane < 16 ? 0 : 32;    // its half of the columns
        auto read_state = [&](float (&f)[32], float& zv) {
            uint32_t r[32];
            tmem_ld16x2<32>(tmem + CF::COL_S + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
            tmem_ld16x2<32>(tmem + CF::COL_S + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
            uint32_t zr[16];
            tmem_ld16(tmem + CF::COL_Z + lane_base, zr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(r[e]);
            zv = __uint_as_float(zr[0]);
        };
        // S_k, z_k -> bf16 operands (buffer k & 1): row a of S, z as hi + lo rows
        auto write_operands = [&](int k, const float (&f)[32], float zv) {
            uint8_t* b3b = b3 + (k & 1) * CF::B3;
#pragma unroll
            for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4*>(b3b + sw128_off(a, cb + 8 * g)) = pack8(f + 8 * g);
            if (normalize && lane < 16) {
                const __nv_bfloat16 hi = __float2bfloat16_rn(zv);
                const __nv_bfloat16 lo = __float2bfloat16_rn(zv - __bfloat162float(hi));
                uint8_t* bzb = bz + (k & 1) * CF::BZ;
                *reinterpret_cast<__nv_bfloat16*>(bzb + sw128_off(0, a)) = hi;
                *reinterpret_cast<__nv_bfloat16*>(bzb + sw128_off(1, a)) = lo;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(bprep);
        };
        // phase A
        for (int ld = 0; ld < nsub; ++ld) transform_k(ld);
        mbar_wait(bsdone, 0, err);
        tc_fence_after();
        {
            float f[32], zv;
            read_state(f, zv);
            if (PHI == PHI_RELU1) {
                // + 1 (x) colsum(V) (every row of the P columns holds it) and
                // z = colsum(relu K) + the block's key count
                uint32_t r[32];
                tmem_ld16x2<32>(tmem + CF::COL_P + lane_base, *reinterpret_cast<uint32_t(*)[16]>(r));
                tmem_ld16x2<32>(tmem + CF::COL_P + lane_base + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] += __uint_as_float(r[e]);
                zv += (float)nkeys;
            }
#pragma unroll
            for (int g = 0; g < 8; ++g)
                *reinterpret_cast<float4*>(xch + a * D + cb + 4 * g) = make_float4(f[4 * g], f[4 * g + 1], f[4 * g + 2],
                                                                                   f[4 * g + 3]);
            if (lane < 16) xch[D * D + a] = zv;
        }
        // phase B: the block prefix over the cluster's lower ranks, in rank order
        asm volatile("barrier.cluster.arrive;" ::: "memory");
        asm volatile("barrier.cluster.wait;" ::: "memory");
        phase_b_waited = true;
        float* sbp = reinterpret_cast<float*>(pt);  // staged in the (idle) P~ buffers
        for (int e4 = et; e4 < (D * D + D) / 4; e4 += 128) {
            // the lower ranks' pieces, eight loads in flight, summed in rank order
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r0 = 0; r0 < rank; r0 += 8) {
                float4 x[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (r0 + q < rank) x[q] = ld_cluster_f4(cluster_addr(xch + 4 * e4, r0 + q));
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (r0 + q < rank) {
                        acc.x += x[q].x;
                        acc.y += x[q].y;
                        acc.z += x[q].z;
                        acc.w += x[q].w;
                    }
            }
            reinterpret_cast<float4*>(sbp)[e4] = acc;
            if (S_total != nullptr && rank == (int)gridDim.x - 1) {
                // the head's total (the state a decode continues from)
                const float4 own = reinterpret_cast<const float4*>(xch)[e4];
                const float4 tot = make_float4(acc.x + own.x, acc.y + own.y, acc.z + own.z, acc.w + own.w);
                if (4 * e4 < D * D)
                    reinterpret_cast<float4*>(S_total + (size_t)bh * D * D)[e4] = tot;
                else
                    reinterpret_cast<float4*>(z_total + (size_t)bh * D)[e4 - D * D / 4] = tot;
            }
        }
        named_bar(1, 128);
        {
            // seed the running state with the block prefix; S_0 = S_bp
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = sbp[a * D + cb + e];
            const float zv = sbp[D * D + a];
            // 32x32b stores: lanes 16..31 hold no row of an M = 64 accumulator;
            // write the columns of this thread's half through the two 16-lane halves
            uint32_t r[16];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    r[e] = lane < 16 ? __float_as_uint(sbp[a * D + c0 + e]) : 0u;
                tmem_st16(tmem + CF::COL_S + lane_base + c0, r);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = lane < 16 ? __float_as_uint(zv) : 0u;
            tmem_st16(tmem + CF::COL_Z + lane_base, r);
            tmem_st_wait();
            named_bar(1, 128);  // every read of the staged prefix is done before the mask warps reuse P~
            write_operands(0, f, zv);
        }
        // phase D
        mbar_wait(binned, 0, err);
        for (int k = 0; k < nsub; ++k) {
            transform_k(nsub + k);
            for (int n = step_begin[k]; n < step_begin[k + 1]; ++n) {
                const int op = ops[n];
                if (!op_opens(op)) continue;
                const int t = op_tile(op), qb = t % CF::QB;
                mbar_wait(qfull + qb, (t / CF::QB) & 1, err);
                if (mapped) {
                    constexpr int NL = CF::TILE / 16 / 128;
                    uint4* q = reinterpret_cast<uint4*>(qbuf + qb * CF::TILE);
                    uint4 w[NL];
#pragma unroll
                    for (int j = 0; j < NL; ++j) w[j] = q[et + 128 * j];
#pragma unroll
                    for (int j = 0; j < NL; ++j) q[et + 128 * j] = phi8<PHI>(w[j]);
                    fence_async_smem();
                }
                mbar_arrive(qready + qb);
            }
            if (k + 1 < nsub) {
                mbar_wait(bsdone, (k + 1) & 1, err);
                tc_fence_after();
                float f[32], zv;
                read_state(f, zv);
                write_operands(k + 1, f, zv);
            }
        }
    } else {
        // ---------------- mask + epilogue warps ----------------
        const int mt = threadIdx.x - 192;  // 0..127
        const int mw = mt >> 5;            // mask warp 0..3
        // binning: the queries with m_i in [k0, k0 + nkeys), stably sorted by
        // the sub-block of m_i (each mask warp takes a quarter of the sequence)
        if (CAUSAL) {
            // queries = the block's tokens; tile t = sub-block t, one op each
            if (mt == 0) {
                for (int k = 0; k < nsub; ++k) {
                    step_begin[k] = k;
                    ops[k] = op_pack(k, k, true, true);
                }
                step_begin[nsub] = nsub;
                misc[0] = nkeys;
                misc[1] = nsub;
                misc[2] = nsub;
                mbar_arrive(binned);
            }
        } else {
        // the sequence's m row into shared memory first (the second half of
        // the P~ buffers, idle until phase D), every load in flight at once
        int* mb = reinterpret_cast<int*>(pt + CF::PT);
        {
            // coalesced 4-byte loads (rows of m start anywhere), all issued
            // before the first store
            const int32_t* mg = m + (size_t)b * N;
            constexpr int PER = CF::NMAX / 128;
            int w[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j) w[j] = mt + 128 * j < N ? mg[mt + 128 * j] : 0;
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (mt + 128 * j < N) mb[mt + 128 * j] = w[j];
        }
        for (int c = mt; c < 4 * CF::MAX_SUB; c += 128) hist[c] = 0;
        named_bar(2, 128);
        const int qlen = (N + 3) / 4, i0 = mw * qlen, i1 = min(N, i0 + qlen);
        bool bad = false;
        for (int i = i0 + lane; i < i1; i += 32) {
            int mi = mb[i];
            if (mi < 0 || mi > N - 1) {
                bad = true;
                mi = mi < 0 ? 0 : N - 1;
            }
            if (mi >= k0 && mi < k0 + nkeys) atomicAdd(&hist[mw * CF::MAX_SUB + (mi - k0) / KC], 1);
        }
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0 && rank == 0) atomicOr(err, FLAG_MASK_RANGE);
        named_bar(2, 128);
        if (mt == 0) {
            // bucket c of warp w starts after every earlier bucket and after
            // bucket c of the earlier warps
            int pos = 0;
            for (int c = 0; c < nsub; ++c)
                for (int w = 0; w < 4; ++w) {
                    bbase[w * CF::MAX_SUB + c] = pos;
                    pos += hist[w * CF::MAX_SUB + c];
                }
            misc[0] = pos;
        }
        named_bar(2, 128);
        for (int ib = i0; ib < i1; ib += 32) {
            const int i = ib + lane;
            int mi = i < i1 ? mb[i] : -1;
            mi = min(max(mi, 0), N - 1);
            const bool in = i < i1 && mi >= k0 && mi < k0 + nkeys;
            const int c = in ? (mi - k0) / KC : -1;
            const unsigned act = __ballot_sync(0xffffffffu, in);
            const unsigned same = __match_any_sync(0xffffffffu, c) & act;
            if (in) {
                const int rk = __popc(same & ((1u << lane) - 1u));
                tab[bbase[mw * CF::MAX_SUB + c] + rk] = (i << CF::LIM_BITS) | (mi - k0);
            }
            __syncwarp();
            if (in && lane == __ffs(same) - 1) bbase[mw * CF::MAX_SUB + c] += __popc(same);
            __syncwarp();
        }
        named_bar(2, 128);
        const int nq = misc[0];
        const int nt = (nq + KC - 1) / KC;
        if (mt == 0) {
            // the ops of phase D in order: at sub-block k, the tile carried
            // from k - 1 (if any), then the tiles whose first query lies in k
            int nops = 0, t = 0, carried = -1;
            for (int k = 0; k < nsub; ++k) {
                step_begin[k] = nops;
                if (carried >= 0) {
                    const int last = (tab[min(nq, (carried + 1) * KC) - 1] & ((1 << CF::LIM_BITS) - 1)) / KC;
                    ops[nops++] = op_pack(carried, k, false, last == k);
                    if (last == k) carried = -1;
                }
                while (carried < 0 && t < nt && (tab[t * KC] & ((1 << CF::LIM_BITS) - 1)) / KC == k) {
                    const int last = (tab[min(nq, (t + 1) * KC) - 1] & ((1 << CF::LIM_BITS) - 1)) / KC;
                    ops[nops++] = op_pack(t, k, true, last == k);
                    if (last != k) carried = t;
                    ++t;
                }
            }
            step_begin[nsub] = nops;
            misc[1] = nt;
            misc[2] = nops;
            mbar_arrive(binned);
        }
        }  // !CAUSAL
        asm volatile("barrier.cluster.arrive;" ::: "memory");
        mbar_wait(binned, 0, err);
        const int nops = misc[2];
        // phase D: thread mt owns row mt of every tile
        const int sp = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
        const int i = sp * 32 + lane;  // row of the M = 128 accumulators this thread reads
        float rs[2] = {0.f, 0.f};      // denominator row sums per O slot
        bool ok = true;
        const int nq = misc[0];
        for (int n = 0; n < nops; ++n) {
            const int op = ops[n], t = op_tile(op), k = op_sub(op), j = n & 1, os = t & 1;
            const int pos = t * KC + i;
            // keys 0..lim of sub-block k visible (causal: the diagonal and before)
            const int lim = pos >= nq ? -1 : (CAUSAL ? pos : (tab[pos] & ((1 << CF::LIM_BITS) - 1))) - k * KC;
            ok = mbar_wait(pfull + j, (n >> 1) & 1, err) && ok;
            tc_fence_after();
            uint8_t* ptj = pt + j * CF::PT;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[64];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld16(tmem + CF::COL_P + j * KC + lane_base + 64 * h + 16 * q,
                              *reinterpret_cast<uint32_t(*)[16]>(r + 16 * q));
                tmem_ld_wait();
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = 64 * h + 8 * g + e;
                        f[e] = col <= lim ? __uint_as_float(r[8 * g + e]) : 0.f;
                        rs[os] += f[e];
                    }
                    *reinterpret_cast<uint4*>(ptj + h * CF::TILE + sw128_off(i, 8 * g)) = pack8(f);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(ptready + j);
            if (op_closes(op)) {
                // epilogue: row i of the tile
                ok = ok && mbar_wait(ofull + os, (t >> 1) & 1, err);
                tc_fence_after();
                uint32_t o[D], oz[2];
#pragma unroll
                for (int q = 0; q < D / 16; ++q)
                    tmem_ld16(tmem + CF::COL_O + os * CF::OSLOT + lane_base + 16 * q,
                              *reinterpret_cast<uint32_t(*)[16]>(o + 16 * q));
                tmem_ld2(tmem + CF::COL_O + os * CF::OSLOT + D + lane_base, oz);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(ofree + os);
                const float den = rs[os] + __uint_as_float(oz[0]) + __uint_as_float(oz[1]);
                const float inv = normalize ? __frcp_rn(den) : 1.0f;
                rs[os] = 0.f;
                if (ok && pos < nq) {
                    const int tok = CAUSAL ? k0 + pos : tab[pos] >> CF::LIM_BITS;
                    uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)bh * N + tok) * D);
#pragma unroll
                    for (int g = 0; g < D / 8; ++g) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[8 * g + e]) * inv;
                        dst[g] = pack8(f);
                    }
                }
            }
        }
    }
    if (!phase_b_waited) asm volatile("barrier.cluster.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    // no CTA leaves while a later rank of its cluster may still read its state
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, PfCfg::TMEM_COLS);
    }
}

template <int PHI, bool CAUSAL>
cudaError_t launch_prefix_fused(const Problem& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                const int32_t* m, int block_tokens, int nc, void* out, float* S_total, float* z_total,
                                uint32_t* err, cudaStream_t st) {
    cudaError_t e = ensure_smem<tc_prefix_fused_kernel<PHI, CAUSAL>>(PfCfg::SMEM);
    if (e != cudaSuccess) return e;
    return launch_cluster_pdl(tc_prefix_fused_kernel<PHI, CAUSAL>, dim3(nc, (unsigned)p.bh()), dim3(PfCfg::THREADS),
                              PfCfg::SMEM, st, (unsigned)nc, mq, mk, mv, m, p.H, p.N, block_tokens, p.normalize,
                              static_cast<__nv_bfloat16*>(out), S_total, z_total, err);
}

template <bool CAUSAL>
cudaError_t fused_phi(const Problem& p, const void* q, const void* k, const void* v, const int32_t* m, void* out,
                      float* S_total, float* z_total, uint32_t* err, cudaStream_t st) {
    int bt = 0, nc = 0;
    if (!tc_prefix_fused_plan(p, &bt, &nc)) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mv;
    // causal: Q tiles of the block's own tokens; prefix mask: a 2-D row map for tile::gather4
    cudaError_t e = CAUSAL ? make_map(&mq, q, PfCfg::D, p.N, p.bh(), PfCfg::KC) : make_row_map(&mq, q, PfCfg::D, p.bh() * p.N);
    if (e == cudaSuccess) e = make_map(&mk, k, PfCfg::D, p.N, p.bh(), PfCfg::KC);
    if (e == cudaSuccess) e = make_map(&mv, v, PfCfg::D, p.N, p.bh(), PfCfg::KC);
    if (e != cudaSuccess) return e;
    switch (p.phi) {  // one kernel per feature map (see phi8)
        case PHI_RELU1: return launch_prefix_fused<PHI_RELU1, CAUSAL>(p, mq, mk, mv, m, bt, nc, out, S_total, z_total, err, st);
        case PHI_ELU1: return launch_prefix_fused<PHI_ELU1, CAUSAL>(p, mq, mk, mv, m, bt, nc, out, S_total, z_total, err, st);
        default: return launch_prefix_fused<PHI_IDENTITY, CAUSAL>(p, mq, mk, mv, m, bt, nc, out, S_total, z_total, err, st);
    }
}

}  // namespace

bool tc_prefix_fused_plan(const Problem& p, int* block_tokens, int* nc) {
    if (p.dtype != DT_BF16 || p.d != PfCfg::D || p.N > PfCfg::NMAX) return false;
    // one CTA per SM: as many blocks per head as fill the SMs, at most 8 (a
    // portable cluster), fewer while the heads' clusters would not all be
    // resident at once (a cluster lives inside one GPC)
    for (long long per_head = std::max(1LL, std::min(8LL, (long long)device_sms() / p.bh())); per_head >= 1;
         --per_head) {
        const int bt = (int)(((p.N + per_head - 1) / per_head + PfCfg::KC - 1) / PfCfg::KC * PfCfg::KC);
        const int n = (p.N + bt - 1) / bt;
        if (p.bh() <= max_active_clusters(n, PfCfg::THREADS, PfCfg::SMEM)) {
            *block_tokens = bt;
            *nc = n;
            return true;
        }
    }
    return false;
}

cudaError_t tc_prefix_fused(const Problem& p, const void* q, const void* k, const void* v, const int32_t* m, void* out,
                            uint32_t* err, cudaStream_t st) {
    return fused_phi<false>(p, q, k, v, m, out, nullptr, nullptr, err, st);
}

cudaError_t tc_causal_fused(const Problem& p, const void* q, const void* k, const void* v, void* out, float* S_total,
                            float* z_total, uint32_t* err, cudaStream_t st) {
    return fused_phi<true>(p, q, k, v, nullptr, out, S_total, z_total, err, st);
}

}  // namespace la
