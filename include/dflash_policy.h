/*
 * dflash_policy.h — block-size (gamma) choice between speculative cycles.
 *
 * DFlash technical summary (gist.science ja/nl), §3 contribution 4 and the
 * block-size bullet of the §4 ablations: a drafter trained with large blocks
 * (16) also drafts well with smaller inference blocks, so the block size can
 * be scheduled dynamically.  The summaries give no schedule; this is the plain
 * reading used here, host-side arithmetic only (no CUDA call, no device
 * memory), between one cycle's dflash_accept and the next dflash_draft_block:
 *
 *   Acceptance model.  Each draft position of a block is accepted with the same
 *   probability alpha given that every earlier one was (a geometric acceptance
 *   length, the model the synthetic acceptance plans of the benchmarks follow).
 *   A cycle with block gamma and acceptance length a (0 <= a <= gamma-1, the
 *   value dflash_accept returns) shows a accepted positions and, when
 *   a < gamma-1, one rejected position; when a == gamma-1 the block ran out
 *   before a rejection (censored).
 *   Estimate.  accepts and rejects are running sums over observed cycles, each
 *   call first multiplying both by `decay` (1 keeps everything, 0 keeps only
 *   the newest call); alpha = (accepts + prior_accepts) /
 *   (accepts + rejects + prior_accepts + prior_rejects), which for decay 1 and
 *   vanishing priors is the maximum-likelihood alpha of the censored geometric
 *   model.
 *   Choice.  The expected tokens a cycle commits at block gamma (accepted
 *   drafts plus the target's own next token) are
 *     tau(alpha, gamma) = sum_{k=0}^{gamma-1} alpha^k,
 *   and a cycle is taken to cost cost_fixed + cost_per_token * gamma (any unit:
 *   the drafter's step is nearly flat in gamma at small batch, while the
 *   target's verification grows with it).  The policy returns the candidate
 *   with the largest tau / cost, the smaller gamma on an exact tie.
 *
 * All functions return DFLASH_OK (0) or DFLASH_INVALID_ARG (-1, see dflash.h)
 * and leave the policy unchanged on error.  The struct is plain data owned by
 * the caller (copy it to snapshot the state); one policy serves one stream of
 * cycles (e.g. one batch whose requests share gamma).
 */
#ifndef DFLASH_POLICY_H_
#define DFLASH_POLICY_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DFLASH_POLICY_MAX_CANDIDATES 8

typedef struct {
    int n_candidates;                                  /* 1..DFLASH_POLICY_MAX_CANDIDATES */
    int candidates[DFLASH_POLICY_MAX_CANDIDATES];      /* strictly ascending block sizes, each >= 1 */
    double decay;                                      /* in [0, 1] */
    double cost_fixed, cost_per_token;                 /* >= 0 each, cost > 0 at every candidate */
    double prior_accepts, prior_rejects;               /* > 0 each */
    double accepts, rejects;                           /* running state, start at 0 */
} dflash_gamma_policy;

/* Fill *p (host pointer) with the candidates (host int[n], ascending), the
 * forgetting factor, the cost model and the prior pseudo-counts; the running
 * state starts empty, so the first choice follows the prior alone. */
int dflash_gamma_policy_init(dflash_gamma_policy* p, const int* candidates, int n, double decay, double cost_fixed,
                             double cost_per_token, double prior_accepts, double prior_rejects);

/* Record one cycle of `batch` requests drafted with block `gamma` (>= 1):
 * accept_len is a HOST int32[batch] of acceptance lengths, each in
 * [0, gamma-1] (DFLASH_INVALID_ARG otherwise, nothing recorded). */
int dflash_gamma_policy_observe(dflash_gamma_policy* p, const int32_t* accept_len, int batch, int gamma);

/* The current acceptance estimate alpha (host double out). */
int dflash_gamma_policy_alpha(const dflash_gamma_policy* p, double* alpha);

/* tau(alpha, gamma) = sum_{k<gamma} alpha^k for alpha in [0, 1], gamma >= 1. */
int dflash_gamma_policy_expected_tokens(double alpha, int gamma, double* tau);

/* The candidate with the largest tau(alpha, gamma) / cost(gamma) (host int out). */
int dflash_gamma_policy_choose(const dflash_gamma_policy* p, int* gamma);

#ifdef __cplusplus
}
#endif

#endif /* DFLASH_POLICY_H_ */
