// Draft-length choice from a measured step-latency model (host code only).
//
// The pages leave the draft length to be tuned at inference time ("zero-shot"
// block length, summary 核心方法 / "推理优化 (§3.3)") and name picking it to fit
// the GPU's free token slots as future work (summary, "局限与 Future Work",
// Future work 2).  Here the choice maximises expected tokens per microsecond:
// E(k, alpha) / t(k), with t(k) the measured (or roofline-modelled) step
// latency at draft length k and E the steady-state tokens a step emits when
// each draft is accepted independently with probability alpha.
//
// E follows the decode-step state machine of the library: a step verifies k
// drafts; j* = leading accepts; it emits the accepted drafts that were not
// already emitted plus, if j* < k, the resampled token, which becomes the next
// step's pre-accepted slot 1 (verified without a test).  With m tested slots
// the expected new tokens are e(m) = sum_{i=1..m} alpha^i + (1 - alpha^m);
// from a step without a pre-accepted slot (m = k) the next has one with
// probability 1 - alpha^k, from a step with one (m = k - 1) with probability
// 1 - alpha^(k-1).  E is the average of e(k) and e(k - 1) under the stationary
// distribution of that two-state chain.
#include <cmath>

#include "common.cuh"

namespace {

// Expected new tokens of a step that tests m fresh drafts.
double tokens_of_tests(int m, double alpha) {
    double s = 0.0, a = 1.0;
    for (int i = 1; i <= m; ++i) {
        a *= alpha;
        s += a;
    }
    return s + (1.0 - a);  // a = alpha^m: a resample follows unless all m are accepted
}

}  // namespace

extern "C" {

double tidar_expected_tokens_per_step(int k, double alpha) {
    if (k < 1 || k > tidar::kMaxDraft || !(alpha >= 0.0 && alpha <= 1.0)) return -1.0;
    const double ak = std::pow(alpha, k), ak1 = std::pow(alpha, k - 1);
    const double to_pre_from_free = 1.0 - ak;  // a rejection among k tests
    const double stay_free_from_pre = ak1;     // all k-1 tests accepted after a pre-accepted slot
    const double pi_pre = to_pre_from_free / (to_pre_from_free + stay_free_from_pre);
    return (1.0 - pi_pre) * tokens_of_tests(k, alpha) + pi_pre * tokens_of_tests(k - 1, alpha);
}

int tidar_pick_draft_length(const double *step_us, int n, double alpha, double *tokens_per_us) {
    if (!step_us || n < 1 || n > tidar::kMaxDraft || !(alpha >= 0.0 && alpha <= 1.0)) return 0;
    int best = 0;
    double best_rate = -1.0;
    for (int k = 1; k <= n; ++k) {
        const double t = step_us[k - 1];
        if (!(t > 0.0) || !std::isfinite(t)) continue;  // not measured: not a candidate
        const double rate = tidar_expected_tokens_per_step(k, alpha) / t;
        if (rate > best_rate) {  // ties keep the shorter draft (less work for the same rate)
            best_rate = rate;
            best = k;
        }
    }
    if (tokens_per_us) *tokens_per_us = best ? best_rate : 0.0;
    return best;
}

}  // extern "C"
