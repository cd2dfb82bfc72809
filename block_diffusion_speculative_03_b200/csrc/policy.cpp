// Block-size (gamma) policy between speculative cycles: a geometric acceptance
// estimate with exponential forgetting and the candidate with the most expected
// committed tokens per unit of cycle cost.  Host arithmetic only.
//
// DFlash technical summary (gist.science ja/nl), §3 contribution 4 and the
// block-size ablation bullet of §4: blocks trained at 16 also serve smaller
// inference blocks, so the block size may change from cycle to cycle.
#include <cmath>

#include "dflash.h"
#include "dflash_policy.h"

namespace {

bool finite_nonneg(double v) { return std::isfinite(v) && v >= 0.0; }

bool valid(const dflash_gamma_policy* p) {
    if (!p || p->n_candidates < 1 || p->n_candidates > DFLASH_POLICY_MAX_CANDIDATES) return false;
    for (int i = 0; i < p->n_candidates; ++i) {
        const int g = p->candidates[i];
        if (g < 1 || (i > 0 && g <= p->candidates[i - 1])) return false;
        if (!(p->cost_fixed + p->cost_per_token * g > 0.0)) return false;
    }
    return std::isfinite(p->decay) && p->decay >= 0.0 && p->decay <= 1.0 && finite_nonneg(p->cost_fixed) &&
           finite_nonneg(p->cost_per_token) && std::isfinite(p->prior_accepts) && p->prior_accepts > 0.0 &&
           std::isfinite(p->prior_rejects) && p->prior_rejects > 0.0 && finite_nonneg(p->accepts) &&
           finite_nonneg(p->rejects);
}

// sum_{k<gamma} alpha^k, added term by term (no 1 - alpha cancellation near 1).
double expected_tokens(double alpha, int gamma) {
    double tau = 0.0, term = 1.0;
    for (int k = 0; k < gamma; ++k) {
        tau += term;
        term *= alpha;
    }
    return tau;
}

}  // namespace

extern "C" {

int dflash_gamma_policy_init(dflash_gamma_policy* p, const int* candidates, int n, double decay, double cost_fixed,
                             double cost_per_token, double prior_accepts, double prior_rejects) {
    if (!p || !candidates || n < 1 || n > DFLASH_POLICY_MAX_CANDIDATES) return DFLASH_INVALID_ARG;
    dflash_gamma_policy q = {};
    q.n_candidates = n;
    for (int i = 0; i < n; ++i) q.candidates[i] = candidates[i];
    q.decay = decay;
    q.cost_fixed = cost_fixed;
    q.cost_per_token = cost_per_token;
    q.prior_accepts = prior_accepts;
    q.prior_rejects = prior_rejects;
    if (!valid(&q)) return DFLASH_INVALID_ARG;
    *p = q;
    return DFLASH_OK;
}

int dflash_gamma_policy_observe(dflash_gamma_policy* p, const int32_t* accept_len, int batch, int gamma) {
    if (!valid(p) || !accept_len || batch < 1 || gamma < 1) return DFLASH_INVALID_ARG;
    double acc = 0.0, rej = 0.0;
    for (int b = 0; b < batch; ++b) {
        const int a = accept_len[b];
        if (a < 0 || a > gamma - 1) return DFLASH_INVALID_ARG;
        acc += a;
        rej += (a < gamma - 1) ? 1.0 : 0.0;
    }
    p->accepts = p->decay * p->accepts + acc;
    p->rejects = p->decay * p->rejects + rej;
    return DFLASH_OK;
}

int dflash_gamma_policy_alpha(const dflash_gamma_policy* p, double* alpha) {
    if (!valid(p) || !alpha) return DFLASH_INVALID_ARG;
    const double s = p->accepts + p->prior_accepts;
    *alpha = s / (s + p->rejects + p->prior_rejects);
    return DFLASH_OK;
}

int dflash_gamma_policy_expected_tokens(double alpha, int gamma, double* tau) {
    if (!tau || !std::isfinite(alpha) || alpha < 0.0 || alpha > 1.0 || gamma < 1) return DFLASH_INVALID_ARG;
    *tau = expected_tokens(alpha, gamma);
    return DFLASH_OK;
}

int dflash_gamma_policy_choose(const dflash_gamma_policy* p, int* gamma) {
    double alpha;
    if (!gamma || dflash_gamma_policy_alpha(p, &alpha) != DFLASH_OK) return DFLASH_INVALID_ARG;
    int best = p->candidates[0];
    double best_rate = -1.0;
    for (int i = 0; i < p->n_candidates; ++i) {   // ascending: a strict improvement is needed to move up
        const int g = p->candidates[i];
        const double rate = expected_tokens(alpha, g) / (p->cost_fixed + p->cost_per_token * g);
        if (rate > best_rate) {
            best_rate = rate;
            best = g;
        }
    }
    *gamma = best;
    return DFLASH_OK;
}

}  // extern "C"
