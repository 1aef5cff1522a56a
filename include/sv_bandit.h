/*
 * sv_bandit.h -- online draft selection for speculative decoding, the host
 * side of the verifier library (libspecverify.so).
 *
 * "FlashSpec: Adaptive Speculative Decoding with Online Bandit Draft
 * Selection and Triton-Optimised Verification", Methodology s.2: the choice
 * of draft model before each decoding step is a K-armed bandit whose reward
 * is the step's fraction of accepted draft tokens; the policy sees only the
 * acceptance history, so it does not change the law of the generated tokens.
 * Two policies:
 *   SV_BANDIT_UCB1      every arm once in index order, then the largest
 *                       mean reward + sqrt(2 ln n / n_j) (Auer, Cesa-Bianchi,
 *                       Fischer 2002); ties to the lower index.
 *   SV_BANDIT_THOMPSON  the largest of per-arm Beta(S_j + 1, F_j + 1) draws;
 *                       a reward r in [0, 1] counts as a success with
 *                       probability r (Agrawal, Goyal 2012); ties to the lower
 *                       index.
 * Randomness (Thompson only): Philox4x32-10 keyed by `seed`, counter
 * (c0, round, slot, tag << 24); the Beta draws of select call number t use
 * round t and tag 5 (slots 2j, 2j + 1 for the two Gamma variates of arm j,
 * Marsaglia-Tsang with Box-Muller normals), the success trial of update call
 * number t uses round t, slot j and tag 6.  A uniform is (2m + 1) 2^-53 with
 * m the top 52 bits of two Philox words (the round counters wrap modulo
 * 2^32).  Results are therefore a function of (K, policy, seed, the sequence
 * of calls).
 *
 * Memory and threads: a handle owns its state (O(K) bytes, no device
 * memory); calls on one handle are serialised internally.  Errors return a
 * non-zero sv_status (spec_verify.h) and set spec_verify_last_error().
 */
#ifndef SV_BANDIT_H
#define SV_BANDIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { SV_BANDIT_UCB1 = 0, SV_BANDIT_THOMPSON = 1 };
#define SV_BANDIT_MAX_ARMS 1024

typedef struct sv_bandit sv_bandit;

/* A selector over K arms (1 <= K <= SV_BANDIT_MAX_ARMS); NULL on a bad
 * argument or allocation failure. */
sv_bandit* sv_bandit_create(int K, int policy, uint64_t seed);
void sv_bandit_destroy(sv_bandit* h);

/* The arm for the next step. */
int sv_bandit_select(sv_bandit* h, int* out_arm);

/* Record reward `reward` (in [0, 1]) for `arm`. */
int sv_bandit_update(sv_bandit* h, int arm, double reward);

/* Record a verified step's outcome for `arm`: the reward is the mean of
 * accept_len[b] / gamma over the sequences with accept_len[b] >= 0 (HOST
 * array of B values, e.g. spec_verify's out_accept_len copied back); a step
 * with no valid sequence records nothing. */
int sv_bandit_update_accept(sv_bandit* h, int arm, const int32_t* accept_len, int B, int gamma);

/* Per-arm pulls and reward sums (arrays of K; either may be NULL). */
int sv_bandit_stats(sv_bandit* h, int64_t* pulls, double* reward_sum);

#ifdef __cplusplus
}
#endif
#endif /* SV_BANDIT_H */
