/*
 * sv_oracle.h -- CPU oracle for batched speculative-sampling verification.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded C
 * restatement of what the verification path computes, used by the tests, by
 * the package's smoke check and by the benchmark's CPU-baseline leg.  It
 * shares no code, header, table or constant with the CUDA library; the product
 * path never links, loads or calls it.
 *
 * Sources (page title, section):
 *   [FS]  "FlashSpec: Adaptive Speculative Decoding with Online Bandit Draft
 *         Selection and Triton-Optimised Verification", Methodology s.1
 *         (on-device verification: temperature before log-softmax, log-space
 *         arithmetic, two log-prob scalars per candidate, on-device
 *         accept/reject) and s.3 (KS distribution gate).
 *   [FD]  "FlexDraft", Problem definition (bonus token sampled at the first
 *         rejection point).
 *   [SSD] "Speculative Speculative Decoding", Technical summary s.2 "Saguaro
 *         sampling" (residual r(.) proportional to max(p_target - p_draft, 0)).
 *   [GBV] "SpecTr-GBV: Multi-Draft Block Verification Accelerating Speculative
 *         Decoding", Methodology, Algorithm 1 (tau, rejected-sub-block set H,
 *         per-draft sub-block verification, target/residual correction).
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 *         Easy as 1, 2, 3", SC'11.
 *
 * Floating point: inputs are fp32 or bf16 (bf16 is widened exactly).  The
 * temperature division and the shift by the row maximum are fp32 operations
 * (that is how a logit tensor is scaled); every sum, log, exp and ratio after
 * that is fp64.
 */
#ifndef SV_ORACLE_H
#define SV_ORACLE_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { SVO_F32 = 0, SVO_BF16 = 1 };

/* Philox counter tags: the 4th counter word is (tag << 24) | (k << 12) | pos. */
enum {
  SVO_TAG_ACCEPT = 1,      /* single-draft acceptance uniform             */
  SVO_TAG_GUMBEL = 2,      /* single-draft residual / bonus Gumbel noise   */
  SVO_TAG_MD_ETA = 3,      /* multi-draft sub-block acceptance uniform     */
  SVO_TAG_MD_GUMBEL = 4,   /* multi-draft correction Gumbel noise          */
  SVO_TAG_GROUP = 7        /* single-draft group-level race noise          */
};

/* Vocabulary entries per group of the single-draft two-level race (group g
 * holds entries [g * SVO_RACE_GROUP, (g + 1) * SVO_RACE_GROUP) of the row). */
enum { SVO_RACE_GROUP = 1024 };

/* Per-sequence tie flags written to out_tie[b]. */
enum {
  SVO_TIE_BERNOULLI = 1,   /* some accept decision had |u - h| < 1e-6      */
  SVO_TIE_GUMBEL = 2       /* the sampled token's top-2 score gap < 1e-4   */
};

/* ---- Philox4x32-10 and the uniform conversions ------------------------ */
void svo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* U[0,1) = (x >> 8) * 2^-24 (accept / eta uniforms). */
double svo_u01_accept(uint32_t x);
/* U(0,1) = (2*(x >> 9) + 1) * 2^-24 (Gumbel uniforms; odd multiples of 2^-24). */
double svo_u01_gumbel(uint32_t x);
/* Raw 32-bit word of the keyed stream: key = (lo32(seed), hi32(seed)),
 * counter = (c0, b, lo32(step), (tag<<24)|(k<<12)|pos), word index w in 0..3. */
uint32_t svo_stream_word(uint64_t seed, uint64_t step, uint32_t tag, uint32_t b,
                         uint32_t k, uint32_t pos, uint32_t c0, uint32_t w);

/* ---- randomness interface ---------------------------------------------
 * The verification algorithm draws randomness in exactly two ways: a
 * Bernoulli(h) event and a draw from a categorical distribution given by
 * unnormalised log-weights.  The default source (rng == NULL) implements them
 * with Philox uniforms: u < h, and Gumbel-max.  Tests may substitute another
 * source (e.g. an exact enumerator).  `gap` receives the tie distance that
 * the default source measures (|u - h|, or the top-2 score gap); other
 * sources may leave it untouched. */
typedef struct svo_rng {
  void* ctx;
  int (*coin)(void* ctx, double h, uint32_t tag, uint32_t b, uint32_t k,
              uint32_t pos, double* gap);
  int64_t (*categorical)(void* ctx, const double* logw, int64_t V, uint32_t tag,
                         uint32_t b, uint32_t pos, double* gap);
} svo_rng;

/* ---- building blocks ------------------------------------------------- */
float svo_bf16_to_f32(uint16_t bits);
/* lp[v] = log_softmax(z / T)[v] per the row definition above.  Returns 0, or
 * -1 when the row maximum is not finite (NaN, +inf, or all -inf). */
int svo_row_logprobs(const void* row, int64_t V, int dtype, float T, double* lp);
/* First index of the maximum raw logit (T = 0 rows).  -1 if max not finite. */
int64_t svo_row_argmax(const void* row, int64_t V, int dtype);
/* log max(p - q, 0) for each v (unnormalised residual log-weight); -inf where
 * p <= q.  Returns the number of v with p > q. */
int64_t svo_residual_logw(const double* lp, const double* lq, int64_t V, double* out);
/* Default Gumbel-max draw over logw with the keyed Philox stream. */
int64_t svo_gumbel_argmax(const double* logw, int64_t V, uint64_t seed, uint64_t step,
                          uint32_t tag, uint32_t b, uint32_t pos, double* gap);

/* Two-level exponential race over logw: group g (SVO_RACE_GROUP entries)
 * has weight W_g = sum of exp(logw) over its entries and exponential
 * E_g = -ln U_g, U_g from word 0 of the keyed block (c0 = g) with tag
 * SVO_TAG_GROUP; the winning group is argmax ln W_g - ln E_g (ties: lowest g);
 * within it the entry is argmax logw_v - ln E_v with the entry noise of
 * svo_gumbel_argmax (tag `tag`).  Returns -1 when every weight is zero.
 * gap = the smaller of the two top-2 score gaps. */
int64_t svo_group_race(const double* logw, int64_t V, uint64_t seed, uint64_t step,
                       uint32_t tag, uint32_t b, uint32_t pos, double* gap);

/* ---- single-draft verification ---------------------------------------
 * target [B, gamma+1, V], draft [B, gamma, V] (dtype), tokens [B, gamma],
 * temps [B].  Processes sequences b in [b_begin, b_end).  Outputs (indexed
 * by absolute b): accept_len [B] (-1 for an invalid sequence), tokens
 * [B, gamma+1] (-1 padded), lp/lq [B, gamma] fp64 (may be NULL; NaN at T = 0
 * and for invalid sequences), tie [B] flags (may be NULL).  Returns 0, or -1
 * on a bad argument. */
int svo_verify(const void* target, const void* draft, const int32_t* tokens,
               const float* temps, int64_t B, int gamma, int64_t V, int dtype,
               uint64_t seed, uint64_t step, int64_t b_begin, int64_t b_end,
               int32_t* out_accept_len, int32_t* out_tokens, double* out_lp,
               double* out_lq, uint8_t* out_tie, const svo_rng* rng);

/* ---- multi-draft (SpecTr-GBV style) verification ---------------------
 * target [B, L+1, V], draft [B, L, V] shared by the K drafts, tokens
 * [B, K, L], temps [B].  Outputs: accept_len [B] (tau, -1 invalid), tokens
 * [B, L+1], draft_index [B] (-1 when tau == 0; may be NULL), tie [B]. */
int svo_verify_multidraft(const void* target, const void* draft, const int32_t* tokens,
                          const float* temps, int64_t B, int K, int L, int64_t V,
                          int dtype, uint64_t seed, uint64_t step, int64_t b_begin,
                          int64_t b_end, int32_t* out_accept_len, int32_t* out_tokens,
                          int32_t* out_draft_index, uint8_t* out_tie, const svo_rng* rng);

/* The same verification with a row set per draft when per_draft != 0:
 * target [B, K, L+1, V] and draft [B, K, L, V], where row (k, i) holds the
 * target / draft logits after draft k's own prefix x_k[0..i) (the
 * prefix-conditioned use of the method; rows of drafts that share a prefix
 * are then equal).  Draft k is weighed with its own rows; the residual law
 * starts from row (0, 0) (every draft shares the empty prefix) and, after an
 * advance, comes from the accepted draft's rows.  per_draft == 0 is
 * svo_verify_multidraft. */
int svo_verify_multidraft_rows(const void* target, const void* draft, const int32_t* tokens,
                               const float* temps, int64_t B, int K, int L, int64_t V,
                               int dtype, int per_draft, uint64_t seed, uint64_t step,
                               int64_t b_begin, int64_t b_end, int32_t* out_accept_len,
                               int32_t* out_tokens, int32_t* out_draft_index,
                               uint8_t* out_tie, const svo_rng* rng);

/* ---- draft selection bandit ([FS] Methodology s.2) -------------------
 * Rewards are fractions of accepted draft tokens, in [0, 1].
 * svo_bandit_uniform: uniform in (0, 1) from Philox block (c0, round, slot,
 *   tag << 24), word pair 0-1 (half = 0) or 2-3 (half = 1).
 * svo_gamma_sample: Gamma(alpha, 1), alpha >= 1 (Marsaglia-Tsang), NaN for
 *   alpha < 1.  svo_beta_sample: X / (X + Y), X ~ Gamma(a) on slot 2 arm,
 *   Y ~ Gamma(b) on slot 2 arm + 1.
 * svo_ucb1_select: UCB1 arm for pulls[K] and reward sums[K] (-1 on bad args).
 * svo_thompson_select: Thompson arm for successes / failures [K] at `round`;
 *   theta[K] (may be NULL) receives the Beta draws.
 * svo_thompson_trial: 1 if a reward counts as a success at update `round`. */
double svo_bandit_uniform(uint64_t seed, uint32_t c0, uint32_t round, uint32_t slot, uint32_t tag,
                          int half);
double svo_gamma_sample(double alpha, uint64_t seed, uint32_t round, uint32_t slot);
double svo_beta_sample(double a, double b, uint64_t seed, uint32_t round, uint32_t arm);
int svo_ucb1_select(int K, const int64_t* pulls, const double* reward_sum);
int svo_thompson_select(int K, const int64_t* succ, const int64_t* fail, uint64_t seed,
                        uint32_t round, double* theta);
int svo_thompson_trial(double reward, uint64_t seed, uint32_t round, uint32_t arm);

#ifdef __cplusplus
}
#endif
#endif /* SV_ORACLE_H */
