// Work plans: pure functions of the problem and the device's SM count, shared
// by workspace sizing (la_workspace_size) and the launches, so that a
// workspace sized for a device always fits what the launches on that device
// use. Host C++ only (no device code), so a host test can check them for any
// SM count.
#pragma once

#include <algorithm>

#include "internal.h"

namespace la {
namespace plan {

// Tokens per tile of the tensor-core KV summary, readout and gradient sweeps
// (tc::kTile; tc_kv.cu checks that the two agree).
constexpr int kTileTokens = 128;

inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline long long round_up(long long x, long long a) { return (x + a - 1) / a * a; }

// Split of the KV summary that is not balanced across heads (CUDA cores,
// fp32 tensor cores): nsplit splits per head of tps tokens each (a multiple
// of 128; the last split may be shorter), at most two CTAs per SM in all
// (one wave of two-per-SM kernels) unless the heads alone are more.
struct SplitPlan {
    int nsplit, tps;
};
inline SplitPlan kv_plan(const Problem& p, int sms) {
    const long long target = std::max(1LL, 2LL * sms / p.bh());
    const long long max_splits = std::max(1LL, cdiv(p.N, 256));
    long long ns = std::min(target, max_splits);
    const long long tps = round_up(cdiv(p.N, ns), 128);
    ns = cdiv(p.N, tps);
    return SplitPlan{(int)ns, (int)tps};
}

// Blocks of the chunked forms: every (block, head) is one CTA of the chunk
// sweep, so the block count per head is chosen to fill one wave (CTAs an SM
// holds at once x SMs) without spilling into a second. Blocks hold at least
// 256 tokens, in multiples of 128.
struct BlockPlan {
    int block_tokens, nblk;
};
// The d = 128 sweeps (tensor-core and CUDA-core alike) hold one CTA per SM
// (shared memory and TMEM); the others two.
inline int sweep_ctas_per_sm(const Problem& p) { return p.d == 128 ? 1 : 2; }
inline BlockPlan block_plan(const Problem& p, int sms) {
    const long long target = std::max(1LL, (long long)sweep_ctas_per_sm(p) * sms / p.bh());
    long long bt = round_up(cdiv(p.N, target), 128);
    bt = std::max(bt, 256LL);
    return BlockPlan{(int)bt, (int)cdiv(p.N, bt)};
}

// Balanced split of the tensor-core KV summary, readout and non-causal
// gradients: a 1-D grid of G CTAs cuts the flattened sequence of (head,
// 128-token tile) pairs into G contiguous ranges of equal length (CTA c
// takes tiles [c*total/G, (c+1)*total/G)). A range that touches several heads
// writes one partial record per head; slot (cta * K + j) holds the record of
// the j-th head the CTA touches.
struct KvBalanced {
    int G, K, tph;    // CTAs, record slots per CTA, tiles per head
    long long total;  // bh * tph
};
// CTAs of a balanced split: one range per resident CTA (per_sm per SM), no
// more ranges than tiles.
inline int balanced_ctas(long long total, int sms, int per_sm) {
    return (int)std::max(1LL, std::min<long long>(total, (long long)sms * per_sm));
}
inline KvBalanced kv_balanced_plan(const Problem& p, int sms, int per_sm = 1) {
    KvBalanced w;
    w.tph = (int)cdiv(p.N, kTileTokens);
    w.total = p.bh() * w.tph;
    w.G = balanced_ctas(w.total, sms, per_sm);
    const long long per = cdiv(w.total, w.G);  // most tiles a CTA gets
    // a range of `per` tiles touches at most ceil(per / tph) + 1 heads
    w.K = (int)std::min<long long>(p.bh(), cdiv(per, w.tph) + 1);
    return w;
}

// Non-causal heads at d <= 32 answered in one launch, one CTA per head (the
// KV sum, then the readout, each a loop over the head's tokens in its CTA):
// heads of at most 256 tokens, whose three-launch form is all fixed cost.
// Longer heads take the split partials, their reduction and the readout,
// which spreads a head's queries over many CTAs.
inline bool small_noncausal(const Problem& p, int sms) {
    (void)sms;
    return p.d <= 32 && p.N <= 256;
}

}  // namespace plan
}  // namespace la
