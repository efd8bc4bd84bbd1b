// Host check of the library's work plans (plan.h) for any SM count: every
// plan must cover its tokens exactly, with no empty piece, and never ask for
// more CTAs or record slots than the sizing gave. Prints one line per
// violation and "checked <n>" at the end; exit status 1 on any violation.
//
// Built and run by tests/test_plans.py with g++ (no GPU, no CUDA runtime
// call: plan.h is plain host code).

#include <cstdio>
#include <cstdlib>
#include <string>
#include <vector>

#include "plan.h"

using la::Problem;
namespace plan = la::plan;

static int g_bad = 0;
static long long g_checked = 0;

#define EXPECT(cond, ...)                                         \
    do {                                                          \
        if (!(cond)) {                                            \
            ++g_bad;                                              \
            std::printf("FAIL %s: ", #cond);                      \
            std::printf(__VA_ARGS__);                             \
            std::printf("\n");                                    \
        }                                                         \
    } while (0)

static void check_split(const Problem& p, int sms) {
    const plan::SplitPlan s = plan::kv_plan(p, sms);
    EXPECT(s.nsplit >= 1 && s.tps >= 128 && s.tps % 128 == 0, "kv_plan N=%d bh=%lld sms=%d", p.N, p.bh(), sms);
    // the splits cover [0, N) and none is empty
    EXPECT((long long)s.nsplit * s.tps >= p.N && (long long)(s.nsplit - 1) * s.tps < p.N,
           "kv_plan cover N=%d nsplit=%d tps=%d sms=%d", p.N, s.nsplit, s.tps, sms);
    // one wave at two CTAs per SM, unless the heads alone are more
    EXPECT((long long)s.nsplit * p.bh() <= 2LL * sms || s.nsplit == 1, "kv_plan wave nsplit=%d bh=%lld sms=%d",
           s.nsplit, p.bh(), sms);
}

static void check_blocks(const Problem& p, int sms) {
    const plan::BlockPlan b = plan::block_plan(p, sms);
    EXPECT(b.block_tokens >= 256 && b.block_tokens % 128 == 0 && b.nblk >= 1, "block_plan N=%d bh=%lld sms=%d", p.N,
           p.bh(), sms);
    EXPECT((long long)b.nblk * b.block_tokens >= p.N && (long long)(b.nblk - 1) * b.block_tokens < p.N,
           "block_plan cover N=%d bt=%d nblk=%d sms=%d", p.N, b.block_tokens, b.nblk, sms);
    // one wave: no more (block, head) CTAs than the SMs hold, unless every
    // head already has a single block of the minimum length
    const long long ctas = (long long)b.nblk * p.bh();
    EXPECT(ctas <= (long long)plan::sweep_ctas_per_sm(p) * sms || b.nblk == 1 || b.block_tokens == 256,
           "block_plan wave ctas=%lld sms=%d", ctas, sms);
}

static void check_balanced(const Problem& p, int sms, int per_sm) {
    const plan::KvBalanced w = plan::kv_balanced_plan(p, sms, per_sm);
    EXPECT(w.G >= 1 && w.G <= (long long)sms * per_sm && w.G <= w.total, "balanced G=%d sms=%d total=%lld", w.G,
           sms, w.total);
    EXPECT(w.tph == (p.N + 127) / 128 && w.total == p.bh() * w.tph, "balanced tiles N=%d", p.N);
    // CTA c takes tiles [c*total/G, (c+1)*total/G): contiguous, covering,
    // non-empty, and touching at most K heads (its record slots)
    long long prev_hi = 0;
    for (long long c = 0; c < w.G; ++c) {
        const long long lo = c * w.total / w.G, hi = (c + 1) * w.total / w.G;
        EXPECT(lo == prev_hi && hi > lo, "balanced range c=%lld lo=%lld hi=%lld", c, lo, hi);
        const long long heads = (hi - 1) / w.tph - lo / w.tph + 1;
        EXPECT(heads <= w.K, "balanced slots c=%lld heads=%lld K=%d N=%d bh=%lld sms=%d", c, heads, w.K, p.N,
               p.bh(), sms);
        prev_hi = hi;
    }
    EXPECT(prev_hi == w.total, "balanced end %lld of %lld", prev_hi, w.total);
    EXPECT(plan::balanced_ctas(w.total, sms, per_sm) == w.G, "balanced_ctas");
}

// "plan B H N d dtype sms" on the command line: print that block plan as
// "block_tokens nblk" (for the Python mirror in bench.py) and exit.
static int print_block_plan(char** argv) {
    const Problem p{atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), atoi(argv[6]), 0, 1};
    const plan::BlockPlan b = plan::block_plan(p, atoi(argv[7]));
    std::printf("%d %d\n", b.block_tokens, b.nblk);
    return 0;
}

int main(int argc, char** argv) {
    if (argc == 8 && std::string(argv[1]) == "plan") return print_block_plan(argv);
    // one-launch short heads (d <= 32, at most 256 tokens), whatever the SM count
    for (int sms : {148, 132, 16, 1}) {
        EXPECT(plan::small_noncausal(Problem{1, 1, 256, 16, 0, 0, 1}, sms), "sms %d", sms);
        EXPECT(plan::small_noncausal(Problem{4, 80, 1, 32, 1, 0, 1}, sms), "sms %d", sms);
        EXPECT(!plan::small_noncausal(Problem{1, 1, 257, 16, 0, 0, 1}, sms), "sms %d", sms);
        EXPECT(!plan::small_noncausal(Problem{64, 64, 256, 64, 0, 0, 1}, sms), "d = 64, sms %d", sms);
        EXPECT(!plan::small_noncausal(Problem{2, sms, 1024, 32, 0, 0, 1}, sms), "sms %d", sms);
    }
    const std::vector<int> sms_list = {1, 2, 7, 16, 20, 66, 78, 114, 132, 148, 160, 264};
    const std::vector<int> Ns = {1, 2, 127, 128, 129, 255, 256, 257, 1000, 2048, 3000, 4096, 16384, 65537, 131072};
    const std::vector<std::pair<int, int>> BHs = {{1, 1}, {1, 3}, {2, 8}, {4, 16}, {8, 8}, {1, 16}, {64, 32}, {3, 37}};
    for (int sms : sms_list)
        for (int N : Ns)
            for (auto bh : BHs)
                for (int d : {16, 64, 128})
                    for (int dtype : {0, 1}) {
                        const Problem p{bh.first, bh.second, N, d, dtype, 0, 1};
                        check_split(p, sms);
                        check_blocks(p, sms);
                        for (int per_sm : {1, 2}) check_balanced(p, sms, per_sm);
                        ++g_checked;
                    }
    std::printf("checked %lld\n", g_checked);
    return g_bad ? 1 : 0;
}
