// sm_100a building blocks: mbarriers, TMA tensor loads, TMEM allocation and
// tcgen05 MMA / load / store, written as inline PTX.
//
// Shared-memory operand layout used throughout: the 128-byte swizzle. A tile
// is a stack of 128-byte rows; within each group of 8 rows (1024 bytes) the
// 16-byte chunk index of row r is XORed with (r mod 8). TMA writes this
// layout when a tensor map uses CU_TENSOR_MAP_SWIZZLE_128B with a 128-byte
// inner box, and tcgen05.mma reads it through a matrix descriptor with
// layout type SWIZZLE_128B:
//   K-major operand  (rows = M or N index, 64 K elements per row):
//       8-row groups SBO bytes apart; a K step of 16 bf16 is +32 bytes.
//   MN-major operand (rows = K index, 64 M/N elements per row):
//       8-row groups SBO bytes apart (a K step of 16 is +2*SBO),
//       64-element M/N atoms LBO bytes apart.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace la {
namespace tc {

// Error-word bit for an expired bounded wait.
constexpr uint32_t FLAG_TIMEOUT = 2u;
// A bounded wait gives up after this long (ns of %globaltimer).
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
// One try_wait: the thread may be suspended in hardware until the phase
// completes or about `hint_ns` pass, whichever is first.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
// Per-CTA abort flag: set by the first wait that expires. From then on every
// abortable wait of the CTA returns at once, so the warps run through the
// rest of their schedule without waiting and reach every named barrier and
// the final __syncthreads together. Kernels clear it with cta_abort_reset()
// before their first __syncthreads.
__device__ __forceinline__ volatile int* cta_abort() {
    __shared__ int flag;
    return &flag;
}
__device__ __forceinline__ void cta_abort_reset() { *cta_abort() = 0; }

// Waits for the phase with the given parity to complete. The waiting thread
// sleeps in try_wait (no polling); the clock is read only between sleeps.
// Gives up after kWaitTimeoutNs: sets FLAG_TIMEOUT in *err and the CTA's
// abort flag, returns false. An abortable wait also returns false at once
// when the abort flag is set; the end-of-kernel waits for a CTA's own copies
// in flight are not abortable (but still bounded).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err,
                                          bool abortable = true) {
    constexpr uint32_t kHintNs = 100000;
    if (mbar_try_wait(bar, parity, kHintNs)) return true;
    volatile int* ab = cta_abort();
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity, kHintNs)) {
        if (abortable && *ab) return false;
        if (globaltimer() - t0 > kWaitTimeoutNs) {
            atomicOr(err, FLAG_TIMEOUT);
            *ab = 1;
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// 3-D tiled load into shared memory, completing on `bar` (bytes counted).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// Row gather (tile::gather4) through a 2-D map whose box is one row high:
// rows r0..r3, columns c0 .. c0 + box width, land as four consecutive rows
// of the destination (swizzled by address like any tiled load), completing
// on `bar`. c0 obeys the tiled-load rule (c0 * element size a multiple of 16).
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int r0,
                                            int r1, int r2, int r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
        : "memory");
}
// One gathered query tile of C rows x BOXW*NB columns (boxes of 128 bytes:
// 64 bf16 or 32 fp32 columns), issued by a whole warp:
// lane l holds the token indices of rows (C/32)*l .. (C/32)*l + C/32 - 1 in
// tok[] (-1 for a padding row, which fetches token 0 instead), and lanes
// 0 .. NB*C/4 - 1 each issue one gather4 of four rows of one box.
// `dst` is the 1024-byte aligned tile, one [C x BOXW] box after another;
// `row0` is the map row of token 0 of the head. The caller posts the
// expected bytes (C * 128 * NB) on `bar` before calling.
template <int C, int NB, int BOXW = 64>
__device__ __forceinline__ void gather_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row0,
                                            const int (&tok)[C / 32], int lane) {
    constexpr int R = C / 32, G = C / 4;  // rows per lane, gathers per box
    static_assert(NB * G <= 32, "one gather per lane");
    const int g = lane % G;
    int r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = __shfl_sync(0xffffffffu, tok[e % R], (4 * g + e) / R);
    if (lane < NB * G) {
        const int bx = lane / G;
        tma_gather4(dst + bx * (C * 128) + g * 512, map, bar, bx * BOXW, row0 + max(r[0], 0), row0 + max(r[1], 0),
                    row0 + max(r[2], 0), row0 + max(r[3], 0));
    }
}
// 3-D tiled store from shared memory (bulk group). Parts of the box outside
// the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
        "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the shared-memory sources of this thread's bulk stores may be
// reused (the stores may still be in flight to global memory).
__device__ __forceinline__ void bulk_wait_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA / tcgen05) accesses.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMEM and tcgen05
// ---------------------------------------------------------------------------
// Whole warp: allocates `ncols` columns (power of 2, >= 32) and writes the
// base address to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;  // descriptor version for sm_100
    d |= 2ull << 61;  // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
// a_mn / b_mn: operand is MN-major (else K-major).
constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                         // D format f32
           | (1u << 7) | (1u << 10)          // A, B format bf16
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D (TMEM) = A * B (+ D when accumulate != 0). Issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on `bar` once every MMA this thread issued before has completed.
// Same, with the A operand read from TMEM instead of shared memory: M lanes
// from the address's lane, K-major, two 16-bit elements per 32-bit column
// (the lower k in the low half), K / 2 columns per instruction.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Warp-wide: lane i receives TMEM lane (base lane + i), 16 consecutive
// 32-bit columns starting at the address's column.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%"
        "15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Warp-wide, for M = 64 accumulators (rows in lanes 0..15 of a
// sub-partition): lanes 0..15 receive TMEM lane (base + i), columns
// [col, col + 16); lanes 16..31 receive TMEM lane (base + i - 16), columns
// [col + SPLIT, col + SPLIT + 16).
template <int SPLIT>
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16], %17;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr), "n"(SPLIT));
}
// Warp-wide, one column of an M = 64 accumulator: lanes 0..15 receive TMEM
// lane (base + i) at the address's column, lanes 16..31 TMEM lane
// (base + i - 16) at column + SPLIT.
template <int SPLIT>
__device__ __forceinline__ void tmem_ld1x2(uint32_t taddr, uint32_t& r) {
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x1.b32 {%0}, [%1], %2;" : "=r"(r) : "r"(taddr), "n"(SPLIT));
}
// Warp-wide: lane i receives TMEM lane (base + i), 2 columns.
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t (&r)[2]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(taddr));
}
// Warp-wide, 16 TMEM lanes, eight repetitions of 8 columns (the 16x256b
// shape): for repetition k, lane i receives in r[4k], r[4k + 1] TMEM lane
// (base + i / 4) at columns col + 8k + 2 (i % 4) + {0, 1}, and in r[4k + 2],
// r[4k + 3] the same columns of TMEM lane (base + 8 + i / 4).
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// Warp-wide: lane i receives TMEM lane (base + i), 4 columns.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Warp-wide: four 8x8 16-bit matrices stored transposed. In register m,
// lane i holds the packed pair (row i / 4, columns 2 (i % 4) and 2 (i % 4) + 1)
// of matrix m; the pair lands in stored rows 2 (i % 4) and 2 (i % 4) + 1 at
// column i / 4. Lanes 8m .. 8m + 7 give the shared addresses of stored rows
// 0..7 of matrix m (16 bytes each, 16-byte aligned).
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t saddr, uint32_t p0, uint32_t p1, uint32_t p2,
                                                  uint32_t p3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(p0),
                 "r"(p1), "r"(p2), "r"(p3)
                 : "memory");
}

// Named barrier over `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

constexpr int kTile = 128;  // tokens per TMA tile of the KV-summary and readout kernels

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ void unpack8(const uint4& w, float* f) { Vec16<__nv_bfloat16>::unpack(w, f); }
__device__ __forceinline__ uint4 pack8(const float* f) { return Vec16<__nv_bfloat16>::pack(f); }

// Byte offset of element (row, col) in a 128-byte-swizzled tile of bf16
// rows, 64 elements per row (col < 64).
__device__ __forceinline__ uint32_t sw128_off(uint32_t row, uint32_t col) {
    return row * 128u + ((((col >> 3) ^ (row & 7u)) << 4) | ((col & 7u) << 1));
}

// phi = relu(x) + 1 on eight packed bf16 values: max(x, 0) then + 1 in
// bf16x2 arithmetic (each result rounded once, as fp32 followed by a round to
// bf16 would give; -0.0 maps to 1 like +0.0).
__device__ __forceinline__ uint4 phi_relu1_x8(uint4 w) {
    const __nv_bfloat162 zero = __float2bfloat162_rn(0.0f), one = __float2bfloat162_rn(1.0f);
    uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v[i]);
        h = __hadd2(__hmax2(h, zero), one);
        v[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
}
// phi = elu(x) + 1 (alpha = 1) on eight packed bf16 values: x + 1 for x > 0,
// exp(x) otherwise, in fp32, each result rounded to bf16 once.
__device__ __forceinline__ uint4 phi_elu1_x8(uint4 w) {
    float f[8];
    unpack8(w, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = f[e] > 0.0f ? f[e] + 1.0f : __expf(f[e]);
    return pack8(f);
}
// The feature map PHI on eight packed bf16 values. The map is a template
// parameter of every tensor-core kernel: with a run-time choice both bodies
// sit inline at every (unrolled) call site, and the larger code ran the d =
// 128 sweep at two thirds of the speed of a single-map build.
template <int PHI>
__device__ __forceinline__ uint4 phi8(uint4 w) {
    if constexpr (PHI == PHI_ELU1) return phi_elu1_x8(w);
    else if constexpr (PHI == PHI_RELU1) return phi_relu1_x8(w);
    else return w;
}
// Bit e of the result is set when element e of eight packed bf16 values is
// greater than zero (sign clear and not +0).
__device__ __forceinline__ uint32_t positive_bits(const uint4& w) {
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = v[i] & 0xFFFFu, hi = v[i] >> 16;
        m |= (((lo & 0x8000u) == 0 && lo != 0) ? 1u : 0u) << (2 * i);
        m |= (((hi & 0x8000u) == 0 && hi != 0) ? 1u : 0u) << (2 * i + 1);
    }
    return m;
}

// f *= phi'(x) on eight values of one row: relu+1 from the sign bits,
// elu+1 from phi(x) itself (packed bf16 in w), the identity leaves f alone.
template <int PHI>
__device__ __forceinline__ void times_phi_grad(float* f, uint32_t bits, const uint4& w) {
    if constexpr (PHI == PHI_RELU1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = ((bits >> e) & 1u) ? f[e] : 0.f;
    } else if constexpr (PHI == PHI_ELU1) {
        float p[8];
        unpack8(w, p);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] *= fminf(p[e], 1.f);
    }
}

// relu on eight packed bf16 values (exact).
__device__ __forceinline__ uint4 relu_x8(uint4 w) {
    const __nv_bfloat162 zero = __float2bfloat162_rn(0.0f);
    uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v[i]);
        h = __hmax2(h, zero);
        v[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Thread-block clusters: distributed shared memory and the cluster barrier
// ---------------------------------------------------------------------------
// Address of `p` (this CTA's shared memory) in the shared memory of cluster
// rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ float ld_cluster_f(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_cluster_f4(uint32_t addr, const float4& v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_u4(uint32_t addr, const uint4& v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void st_cluster_u16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared::cluster.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
// Cluster-wide barrier: arrive (release) then wait (acquire). Every thread of
// every CTA of the cluster takes it, on every path.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive;" ::: "memory");
    asm volatile("barrier.cluster.wait;" ::: "memory");
}

}  // namespace tc
}  // namespace la
