// C ABI of libla_b200 (declared in include/la.h): argument validation,
// workspace planning and kernel dispatch. Validation is fail-closed: a bad
// request returns a status before anything is launched.

#include <la.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "device.h"
#include "internal.h"
#include "launch_util.h"
#include "plan.h"
#include "tc.h"
#include "tc_common.cuh"

namespace la {
namespace {

constexpr int kSimtChunk = 64;     // chunk length the SIMT chunked kernel runs at
constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

la_status check_desc(const la_desc* d) {
    if (d == nullptr) return LA_ERR_INVALID_ARG;
    if (d->B <= 0 || d->H <= 0 || d->N <= 0 || d->d <= 0) return LA_ERR_INVALID_ARG;
    if (d->dtype != LA_F32 && d->dtype != LA_BF16) return LA_ERR_INVALID_ARG;
    if (d->phi != LA_PHI_RELU1 && d->phi != LA_PHI_IDENTITY && d->phi != LA_PHI_ELU1) return LA_ERR_INVALID_ARG;
    if (d->normalize != 0 && d->normalize != 1) return LA_ERR_INVALID_ARG;
    if (d->d != 16 && d->d != 32 && d->d != 64 && d->d != 128) return LA_ERR_UNSUPPORTED;
    if (d->normalize == 1 && d->phi == LA_PHI_IDENTITY) return LA_ERR_UNSUPPORTED;
    if ((long long)d->B * d->H > 65535) return LA_ERR_UNSUPPORTED;  // grid.y limit
    if ((long long)d->B * d->H * d->N * d->d > (1LL << 40)) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

la_status check_chunk(int chunk) { return (chunk == 64 || chunk == 128) ? LA_OK : LA_ERR_UNSUPPORTED; }

// The library's kernels are built for sm_100a only.
la_status check_device() {
    static std::atomic<uint64_t> ok{0}, bad{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    const uint64_t bit = 1ull << (dev & 63);
    if (ok.load() & bit) return LA_OK;
    if (bad.load() & bit) return LA_ERR_UNSUPPORTED;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (major != 10) {
        bad.fetch_or(bit);
        return LA_ERR_UNSUPPORTED;
    }
    ok.fetch_or(bit);
    return LA_OK;
}

Problem to_problem(const la_desc* d) {
    return Problem{d->B, d->H, d->N, d->d, d->dtype, d->phi, d->normalize};
}

// ---- work plans (pure functions of the problem, shared by sizing and launch) ----

// Plans for the current device's SM count (plan.h): a workspace sized on a
// device fits every launch on that device.
plan::SplitPlan kv_plan(const Problem& p) { return plan::kv_plan(p, device_sms()); }
plan::BlockPlan block_plan(const Problem& p) { return plan::block_plan(p, device_sms()); }
using plan::BlockPlan;
using plan::SplitPlan;

int prefix_nbins(const Problem& p, int kchunk) { return p.N / kchunk + 1; }

struct WsLayout {
    size_t part = 0, sz = 0, perm = 0, msort = 0, bins = 0, total = 0;
    size_t grec = 0, gtot = 0, gn = 0, gden = 0;  // gradients
};

WsLayout ws_layout(const Problem& p, int op) {
    WsLayout L;
    size_t off = WS_HEADER;
    const size_t rec = p.state_floats() * sizeof(float);
    if (op == LA_OP_KV_SUMMARY || op == LA_OP_NONCAUSAL) {
        size_t nrec;
        if (tc_supported(p)) {
            const KvBalanced w = kv_balanced_plan(p);
            nrec = (size_t)w.G * w.K;
        } else {
            nrec = (size_t)p.bh() * kv_plan(p).nsplit;
        }
        L.part = off;
        off = round_up(off + nrec * rec, kAlign);
        if (op == LA_OP_NONCAUSAL) {
            L.sz = off;
            off = round_up(off + (size_t)p.bh() * rec, kAlign);
        }
    } else if (op == LA_OP_CAUSAL || op == LA_OP_PREFIX) {
        const BlockPlan bp = block_plan(p);
        L.part = off;
        off = round_up(off + (size_t)p.bh() * bp.nblk * rec, kAlign);
        if (op == LA_OP_PREFIX) {
            const int nbins = prefix_nbins(p, 64);  // the most bins any kernel uses
            L.perm = off;
            off = round_up(off + sizeof(int32_t) * (size_t)p.B * p.N, kAlign);
            L.msort = off;
            off = round_up(off + sizeof(int32_t) * (size_t)p.B * p.N, kAlign);
            L.bins = off;
            off = round_up(off + sizeof(int32_t) * (size_t)p.B * (nbins + 1), kAlign);
        }
    } else if (op == LA_OP_NONCAUSAL_BWD || op == LA_OP_CAUSAL_BWD) {
        const BlockPlan bp = block_plan(p);
        L.part = off;
        if (op == LA_OP_NONCAUSAL_BWD) {
            // the KV summary's own scratch where kv_summary_impl expects it
            // (on the tensor cores it then takes the gradient kernels' (G, h)
            // records, whose split may have more slots), then the totals
            // (S, z) and (G, h)
            off = ws_layout(p, LA_OP_KV_SUMMARY).total;
            if (tc_supported(p)) off = std::max(off, round_up(L.part + tc_backward_record_slots(p) * rec, kAlign));
            L.sz = off;
            off = round_up(off + (size_t)p.bh() * rec, kAlign);
            L.gtot = off;
            off = round_up(off + (size_t)p.bh() * rec, kAlign);
            if (tc_supported(p)) {  // the CUDA-core path's block states and gn, gden are not used
                L.total = off;
                return L;
            }
        } else {
            off = round_up(off + (size_t)p.bh() * bp.nblk * rec, kAlign);  // block states (S, z)
        }
        L.grec = off;
        off = round_up(off + (size_t)p.bh() * bp.nblk * rec, kAlign);      // block states (G, h)
        L.gn = off;
        off = round_up(off + sizeof(float) * (size_t)p.bh() * p.N * p.d, kAlign);
        L.gden = off;
        off = round_up(off + sizeof(float) * (size_t)p.bh() * p.N, kAlign);
    } else {
        return L;
    }
    L.total = off;
    return L;
}

template <typename P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

la_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return LA_OK;
    cudaGetLastError();
    return LA_ERR_CUDA;
}

la_status check_ws(const WsLayout& L, void* ws, size_t ws_bytes) {
    if (ws == nullptr || ws_bytes < L.total) return LA_ERR_WORKSPACE;
    if (!aligned16(ws)) return LA_ERR_MISALIGNED;
    return LA_OK;
}

#define LA_TRY(expr)                      \
    do {                                  \
        la_status s__ = (expr);           \
        if (s__ != LA_OK) return s__;     \
    } while (0)

la_status kv_summary_impl(const Problem& p, const void* k, const void* v, float* S, float* z,
                          void* ws, cudaStream_t st) {
    float* part = at<float>(ws, ws_layout(p, LA_OP_KV_SUMMARY).part);
    if (tc_noncausal_fused_supported(p))  // small problems: one launch, reduced in a cluster per head
        return cuda_status(tc_noncausal_fused(p, nullptr, k, v, nullptr, S, z, at<uint32_t>(ws, 0), st));
    if (tc_supported(p)) return cuda_status(tc_kv_summary(p, k, v, part, S, z, at<uint32_t>(ws, 0), st));
    const SplitPlan sp = kv_plan(p);
    if (tc_f32_supported(p)) {
        LA_TRY(cuda_status(tc_f32_states(p, k, v, sp.tps, sp.nsplit, part, at<uint32_t>(ws, 0), st)));
    } else {
        LA_TRY(cuda_status(simt_kv_partial(p, k, v, sp.tps, sp.nsplit, part, st)));
    }
    return cuda_status(state_reduce(p, part, sp.nsplit, S, z, st));
}

}  // namespace

la_status kv_summary_args(const la_desc* desc, const void* k, const void* v, const float* S_out,
                          const float* z_out) {
    LA_TRY(check_desc(desc));
    if (!k || !v || !S_out || !z_out) return LA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(S_out) || !aligned16(z_out)) return LA_ERR_MISALIGNED;
    return LA_OK;
}

la_status kv_summary_checked(const la_desc* desc, const void* k, const void* v, float* S_out,
                             float* z_out, void* ws, size_t ws_bytes, cudaStream_t st) {
    LA_TRY(kv_summary_args(desc, k, v, S_out, z_out));
    const Problem p = to_problem(desc);
    LA_TRY(check_ws(ws_layout(p, LA_OP_KV_SUMMARY), ws, ws_bytes));
    LA_TRY(check_device());
    timing_begin(st);
    return kv_summary_impl(p, k, v, S_out, z_out, ws, st);
}

}  // namespace la

using namespace la;

extern "C" {

int32_t la_version(void) { return 100; }

const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_MISALIGNED: return "LA_ERR_MISALIGNED";
        case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_MASK_RANGE: return "LA_ERR_MASK_RANGE";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    }
    return "LA_ERR_UNKNOWN";
}

size_t la_workspace_size(const la_desc* desc, int32_t op, int32_t chunk) {
    if (check_desc(desc) != LA_OK) return 0;
    if ((op == LA_OP_CAUSAL || op == LA_OP_PREFIX) && check_chunk(chunk) != LA_OK) return 0;
    if (op < LA_OP_KV_SUMMARY || op > LA_OP_CAUSAL_BWD) return 0;
    return ws_layout(to_problem(desc), op).total;
}

la_status la_kv_summary(const la_desc* desc, const void* k, const void* v, float* S_out,
                        float* z_out, void* ws, size_t ws_bytes, void* stream) {
    return la::kv_summary_checked(desc, k, v, S_out, z_out, ws, ws_bytes,
                                  static_cast<cudaStream_t>(stream));
}

la_status la_noncausal(const la_desc* desc, const void* q, const void* k, const void* v, void* out,
                       float* S_out, float* z_out, void* ws, size_t ws_bytes, void* stream) {
    LA_TRY(check_desc(desc));
    if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
    if ((S_out == nullptr) != (z_out == nullptr)) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_MISALIGNED;
    if (S_out && (!aligned16(S_out) || !aligned16(z_out))) return LA_ERR_MISALIGNED;
    const Problem p = to_problem(desc);
    const WsLayout L = ws_layout(p, LA_OP_NONCAUSAL);
    LA_TRY(check_ws(L, ws, ws_bytes));
    LA_TRY(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    timing_begin(st);
    // small problems: one kernel, a thread-block cluster per head (bf16,
    // d = 64) or one CTA per head (d <= 32)
    if (simt_noncausal_small_supported(p))
        return cuda_status(simt_noncausal_small(p, q, k, v, out, S_out, z_out, st));
    if (tc_noncausal_fused_supported(p))
        return cuda_status(tc_noncausal_fused(p, q, k, v, out, S_out, z_out, at<uint32_t>(ws, 0), st));
    float* S = S_out;
    float* z = z_out;
    if (S == nullptr) {
        S = at<float>(ws, L.sz);
        z = S + (size_t)p.bh() * p.d * p.d;
    }
    LA_TRY(kv_summary_impl(p, k, v, S, z, ws, st));
    if (tc_supported(p)) return cuda_status(tc_readout(p, q, S, z, out, at<uint32_t>(ws, 0), st));
    if (tc_f32_supported(p)) {
        const BlockPlan bp = block_plan(p);
        return cuda_status(tc_f32_readout(p, q, S, z, bp.block_tokens, bp.nblk, out, at<uint32_t>(ws, 0), st));
    }
    return cuda_status(simt_readout(p, q, S, z, out, st));
}

}  // extern "C"

namespace la {
namespace {

// Causal outputs; with S_total/z_total (both or neither) also the state after
// the last token, written by the block-state scan.
la_status causal_impl(const la_desc* desc, int32_t chunk, const void* q, const void* k, const void* v,
                      void* out, float* S_total, float* z_total, void* ws, size_t ws_bytes,
                      cudaStream_t st) {
    LA_TRY(check_desc(desc));
    LA_TRY(check_chunk(chunk));
    if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_MISALIGNED;
    if (S_total && (!aligned16(S_total) || !aligned16(z_total))) return LA_ERR_MISALIGNED;
    const Problem p = to_problem(desc);
    const WsLayout L = ws_layout(p, LA_OP_CAUSAL);
    LA_TRY(check_ws(L, ws, ws_bytes));
    LA_TRY(check_device());
    timing_begin(st);
    const BlockPlan bp = block_plan(p);
    float* part = at<float>(ws, L.part);
    // phase 1: per-block states; phase 2: exclusive prefix over blocks (and
    // the total); phase 3: each block's outputs from its prefix state.
    uint32_t* flags = at<uint32_t>(ws, 0);
    if (tc_supported(p) && p.d == 128 && S_total == nullptr && bp.nblk >= 2) {
        // the states of every block but the last (no block's prefix holds
        // it), then the sweep, whose CTAs each sum the states before their
        // block: no scan kernel in between
        LA_TRY(cuda_status(tc_kv_blocks(p, k, v, bp.block_tokens, bp.nblk, part, flags, st, bp.nblk - 1)));
        return cuda_status(tc_chunked_t(p, q, k, v, part, bp.block_tokens, bp.nblk, nullptr, nullptr, nullptr, 0,
                                        out, flags, st, true));
    }
    if (tc_kv_scan_supported(p, bp.block_tokens, bp.nblk)) {  // phases 1 and 2 in one kernel
        LA_TRY(cuda_status(tc_kv_blocks_scan(p, k, v, bp.block_tokens, bp.nblk, part, S_total, z_total, flags, st)));
    } else {
        if (tc_supported(p)) {
            LA_TRY(cuda_status(tc_kv_blocks(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
        } else if (tc_f32_supported(p)) {
            LA_TRY(cuda_status(tc_f32_states(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
        } else {
            LA_TRY(cuda_status(simt_kv_partial(p, k, v, bp.block_tokens, bp.nblk, part, st)));
        }
        LA_TRY(cuda_status(state_exclusive_scan(p, part, bp.nblk, S_total, z_total, st)));
    }
    if (tc_supported(p))
        return cuda_status(tc_chunked(p, chunk, q, k, v, part, bp.block_tokens, bp.nblk, nullptr,
                                      nullptr, nullptr, 0, out, flags, st));
    if (tc_f32_supported(p))
        return cuda_status(tc_f32_chunked(p, q, k, v, part, bp.block_tokens, bp.nblk, out, flags, st));
    return cuda_status(simt_chunked(p, q, k, v, part, bp.block_tokens, bp.nblk, nullptr, nullptr,
                                    nullptr, 0, out, st));
}

// Gradients of the non-causal or causal form (see la.h): states of the
// forward, a forward sweep for dq, gn, gden and per-block (G, h), the
// suffix (causal) or total (non-causal) of (G, h), a reverse sweep for dk, dv.
la_status backward_impl(const la_desc* desc, bool causal, const void* q, const void* k, const void* v,
                        const void* dout, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
    LA_TRY(check_desc(desc));
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return LA_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                            static_cast<const void*>(dv)})
        if (!aligned16(ptr)) return LA_ERR_MISALIGNED;
    const Problem p = to_problem(desc);
    const WsLayout L = ws_layout(p, causal ? LA_OP_CAUSAL_BWD : LA_OP_NONCAUSAL_BWD);
    LA_TRY(check_ws(L, ws, ws_bytes));
    LA_TRY(check_device());
    timing_begin(st);
    const BlockPlan bp = block_plan(p);
    if (bp.block_tokens % bwd_chunk(p) != 0) return LA_ERR_UNSUPPORTED;
    const long long rec = (long long)p.state_floats();
    float* grec = at<float>(ws, L.grec);
    float* gn = at<float>(ws, L.gn);
    float* gden = at<float>(ws, L.gden);
    if (causal) {
        float* part = at<float>(ws, L.part);
        uint32_t* flags = at<uint32_t>(ws, 0);
        if (tc_kv_scan_supported(p, bp.block_tokens, bp.nblk)) {
            LA_TRY(cuda_status(tc_kv_blocks_scan(p, k, v, bp.block_tokens, bp.nblk, part, nullptr, nullptr, flags, st)));
        } else {
            if (tc_supported(p)) {
                LA_TRY(cuda_status(tc_kv_blocks(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
            } else if (tc_f32_supported(p)) {
                LA_TRY(cuda_status(tc_f32_states(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
            } else {
                LA_TRY(cuda_status(simt_kv_partial(p, k, v, bp.block_tokens, bp.nblk, part, st)));
            }
            LA_TRY(cuda_status(state_exclusive_scan(p, part, bp.nblk, nullptr, nullptr, st)));
        }
        const bool tcq = tc_causal_backward_supported(p, bp.block_tokens);
        if (tcq) {  // tensor cores; gn in bf16
            LA_TRY(cuda_status(tc_causal_backward_q(p, q, k, v, dout, part, bp.block_tokens, bp.nblk, dq, gn, gden,
                                                    grec, flags, st)));
        } else {
            LA_TRY(cuda_status(bwd_q(p, true, q, k, v, dout, part, part + (size_t)p.d * p.d, rec, rec,
                                     bp.block_tokens, bp.nblk, dq, gn, gden, grec, st)));
        }
        LA_TRY(cuda_status(state_exclusive_scan(p, grec, bp.nblk, nullptr, nullptr, st, true)));
        if (tcq)
            return cuda_status(tc_causal_backward_kv(p, q, k, v, gn, gden, grec, bp.block_tokens, bp.nblk, dk, dv,
                                                     flags, st));
        return cuda_status(bwd_kv(p, true, q, k, v, gn, gden, grec, grec + (size_t)p.d * p.d, rec, rec,
                                  bp.block_tokens, bp.nblk, dk, dv, st));
    }
    float* S = at<float>(ws, L.sz);
    float* z = S + (size_t)p.bh() * p.d * p.d;
    float* G = at<float>(ws, L.gtot);
    float* h = G + (size_t)p.bh() * p.d * p.d;
    LA_TRY(kv_summary_impl(p, k, v, S, z, ws, st));
    if (tc_supported(p))  // tensor cores: the KV summary's record slots take the (G, h) records
        return cuda_status(tc_noncausal_backward(p, q, k, v, dout, S, z, at<float>(ws, L.part), G, h, dq, dk, dv,
                                                 at<uint32_t>(ws, 0), st));
    LA_TRY(cuda_status(bwd_q(p, false, q, k, v, dout, S, z, (long long)p.d * p.d, p.d, bp.block_tokens,
                             bp.nblk, dq, gn, gden, grec, st)));
    LA_TRY(cuda_status(state_reduce(p, grec, bp.nblk, G, h, st)));
    return cuda_status(bwd_kv(p, false, q, k, v, gn, gden, G, h, (long long)p.d * p.d, p.d, bp.block_tokens,
                              bp.nblk, dk, dv, st));
}

}  // namespace
}  // namespace la

extern "C" {

la_status la_noncausal_backward(const la_desc* desc, const void* q, const void* k, const void* v,
                                const void* dout, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                void* stream) {
    return backward_impl(desc, false, q, k, v, dout, dq, dk, dv, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

la_status la_causal_backward(const la_desc* desc, const void* q, const void* k, const void* v,
                             const void* dout, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                             void* stream) {
    return backward_impl(desc, true, q, k, v, dout, dq, dk, dv, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

la_status la_causal_chunked(const la_desc* desc, int32_t chunk, const void* q, const void* k,
                            const void* v, void* out, void* ws, size_t ws_bytes, void* stream) {
    return causal_impl(desc, chunk, q, k, v, out, nullptr, nullptr, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

la_status la_causal_prefill(const la_desc* desc, int32_t chunk, const void* q, const void* k,
                            const void* v, void* out, float* S_out, float* z_out, void* ws,
                            size_t ws_bytes, void* stream) {
    if (S_out == nullptr || z_out == nullptr) return LA_ERR_INVALID_ARG;
    return causal_impl(desc, chunk, q, k, v, out, S_out, z_out, ws, ws_bytes,
                       static_cast<cudaStream_t>(stream));
}

la_status la_prefix_mask(const la_desc* desc, int32_t chunk, const void* q, const void* k,
                         const void* v, const int32_t* m, void* out, void* ws, size_t ws_bytes,
                         void* stream) {
    LA_TRY(check_desc(desc));
    LA_TRY(check_chunk(chunk));
    if (!q || !k || !v || !m || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(m))
        return LA_ERR_MISALIGNED;
    const Problem p = to_problem(desc);
    if (p.N > (1 << 21)) return LA_ERR_UNSUPPORTED;  // bin table must fit in shared memory
    const WsLayout L = ws_layout(p, LA_OP_PREFIX);
    LA_TRY(check_ws(L, ws, ws_bytes));
    LA_TRY(check_device());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    timing_begin(st);
    const BlockPlan bp = block_plan(p);
    const bool tc = tc_supported(p);
    const int kchunk = tc ? tc_chunk(p, chunk) : kSimtChunk;  // chunk length of the kernel used
    const int nbins = prefix_nbins(p, kchunk);
    uint32_t* flags = at<uint32_t>(ws, 0);
    int32_t* perm = at<int32_t>(ws, L.perm);
    int32_t* msort = at<int32_t>(ws, L.msort);
    int32_t* bins = at<int32_t>(ws, L.bins);
    float* part = at<float>(ws, L.part);
    // the binning reads only m: launched after the KV pass it runs beside it
    // (bin_kernel waits for its predecessor only at its end); the next
    // kernel (the scan, or the sweep when the KV pass scans in-cluster)
    // waits for both
    const bool cscan = tc_kv_scan_supported(p, bp.block_tokens, bp.nblk);
    if (cscan) {
        LA_TRY(cuda_status(tc_kv_blocks_scan(p, k, v, bp.block_tokens, bp.nblk, part, nullptr, nullptr, flags, st)));
    } else if (tc) {
        LA_TRY(cuda_status(tc_kv_blocks(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
    } else if (tc_f32_supported(p)) {
        LA_TRY(cuda_status(tc_f32_states(p, k, v, bp.block_tokens, bp.nblk, part, flags, st)));
    } else {
        LA_TRY(cuda_status(simt_kv_partial(p, k, v, bp.block_tokens, bp.nblk, part, st)));
    }
    LA_TRY(cuda_status(bin_queries(p, m, kchunk, nbins, perm, bins, msort, flags, st)));
    if (!cscan) LA_TRY(cuda_status(state_exclusive_scan(p, part, bp.nblk, nullptr, nullptr, st)));
    if (tc)
        return cuda_status(tc_chunked(p, chunk, q, k, v, part, bp.block_tokens, bp.nblk, perm, bins,
                                      msort, nbins, out, flags, st));
    if (tc_f32_supported(p))  // 64-token chunks, like the CUDA-core kernel
        return cuda_status(tc_f32_prefix(p, q, k, v, part, bp.block_tokens, bp.nblk, perm, bins, msort, nbins, out,
                                         flags, st));
    return cuda_status(simt_chunked(p, q, k, v, part, bp.block_tokens, bp.nblk, perm, bins, msort,
                                    nbins, out, st));
}

la_status la_decode_step(const la_desc* desc, const void* q, const void* k, const void* v, float* S,
                         float* z, void* out, void* stream) {
    if (desc == nullptr) return LA_ERR_INVALID_ARG;
    la_desc d1 = *desc;
    d1.N = 1;  // N is not used by a decode step
    LA_TRY(check_desc(&d1));
    if (!q || !k || !v || !S || !z || !out) return LA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(S) || !aligned16(z) ||
        !aligned16(out))
        return LA_ERR_MISALIGNED;
    LA_TRY(check_device());
    timing_begin(static_cast<cudaStream_t>(stream));
    return cuda_status(decode_step(to_problem(&d1), q, k, v, S, z, out,
                                   static_cast<cudaStream_t>(stream)));
}

la_status la_last_error(void* ws, void* stream, uint32_t* flags_out) {
    if (ws == nullptr) return LA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t host = 0;
    LA_TRY(cuda_status(cudaMemcpyAsync(&host, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, st)));
    LA_TRY(cuda_status(cudaMemsetAsync(ws, 0, sizeof(uint32_t), st)));
    LA_TRY(cuda_status(cudaStreamSynchronize(st)));
    if (flags_out) *flags_out = host;
    if (host & tc::FLAG_TIMEOUT) return LA_ERR_TIMEOUT;
    if (host & FLAG_MASK_RANGE) return LA_ERR_MASK_RANGE;
    return LA_OK;
}

}  // extern "C"
