/*
 * sv_oracle.c -- CPU oracle for batched speculative-sampling verification.
 *
 * TEST INFRASTRUCTURE ONLY (see sv_oracle.h).  Plain single-threaded C, no
 * blocking, no fusion, no reordering beyond the definitions it restates.  The
 * page citations are given per function; readings that the pages leave open
 * are marked "reading:".
 *
 * Parity status of each function:
 *   svo_philox4x32_10 ...... pinned: published known-answer vectors.
 *   svo_row_logprobs ....... pinned: scipy log_softmax of the fp32-scaled row.
 *   svo_row_argmax ......... pinned: numpy argmax.
 *   svo_residual_logw ...... pinned: exact enumeration (output law == target).
 *   svo_gumbel_argmax ...... pinned: Monte-Carlo chi-square against softmax.
 *   svo_verify ............. pinned: exact enumeration, chi-square over 10^6
 *                            seeded trials, KS gate, acceptance identity,
 *                            geometric accept-length law, T = 0 argmax law.
 *   svo_verify_multidraft .. pinned: exact enumeration (K <= 3, L <= 2),
 *                            chi-square, K = L = 1 equals svo_verify's law,
 *                            T = 0 longest-argmax-prefix law.
 */
#include "sv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define BERNOULLI_TIE_BAND 1e-6
#define GUMBEL_TIE_BAND 1e-4
#define MAX_STEPS 64

/* ------------------------------------------------------------------------
 * Philox4x32-10 (Salmon et al., SC'11, section 3.3): a 4-word counter is
 * pushed through 10 rounds; each round multiplies words 0 and 2 by fixed
 * odd constants, splits the 64-bit products into hi/lo halves, and xors the
 * hi halves with the other two counter words and the round key.  The key is
 * bumped by the Weyl constants (golden ratio, sqrt(3)-1) between rounds.
 * ---------------------------------------------------------------------- */
static void philox_round(uint32_t c[4], const uint32_t k[2]) {
  const uint64_t prod0 = (uint64_t)0xD2511F53u * (uint64_t)c[0];
  const uint64_t prod1 = (uint64_t)0xCD9E8D57u * (uint64_t)c[2];
  const uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
  const uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
  const uint32_t n0 = hi1 ^ c[1] ^ k[0];
  const uint32_t n2 = hi0 ^ c[3] ^ k[1];
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

void svo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k[0] += 0x9E3779B9u;
      k[1] += 0xBB67AE85u;
    }
    philox_round(c, k);
  }
  memcpy(out, c, sizeof c);
}

/* Keyed stream, reading of "keyed by (seed, step, row, position)": key is the
 * 64-bit seed, counter words are (c0, b, lo32(step), tag|k|pos). */
uint32_t svo_stream_word(uint64_t seed, uint64_t step, uint32_t tag, uint32_t b,
                         uint32_t k, uint32_t pos, uint32_t c0, uint32_t w) {
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  const uint32_t ctr[4] = {c0, b, (uint32_t)step, (tag << 24) | (k << 12) | pos};
  uint32_t out[4];
  svo_philox4x32_10(ctr, key, out);
  return out[w & 3u];
}

double svo_u01_accept(uint32_t x) { return (double)(x >> 8) * 0x1p-24; }

double svo_u01_gumbel(uint32_t x) { return (double)(2u * (x >> 9) + 1u) * 0x1p-24; }

/* ------------------------------------------------------------------------
 * Row arithmetic.  [FS] Methodology s.1: the temperature is applied to the
 * logits before the log-softmax, and the arithmetic stays in log space.
 * ---------------------------------------------------------------------- */
float svo_bf16_to_f32(uint16_t bits) {
  const uint32_t w = (uint32_t)bits << 16; /* bf16 is the top half of fp32 */
  float f;
  memcpy(&f, &w, sizeof f);
  return f;
}

static size_t elem_size(int dtype) { return dtype == SVO_BF16 ? 2u : 4u; }

static float logit_at(const void* row, int64_t v, int dtype) {
  if (dtype == SVO_BF16) return svo_bf16_to_f32(((const uint16_t*)row)[v]);
  return ((const float*)row)[v];
}

typedef struct {
  float m;     /* max_v fl32(z_v / T)                      */
  double lnS;  /* ln sum_v exp(fl32(fl32(z_v / T) - m))    */
} row_stat;

/* s_v = fl32(z_v / T); m = max s_v; S = sum exp(fl32(s_v - m)) in fp64. */
static int row_stats(const void* row, int64_t V, int dtype, float T, row_stat* st) {
  float m = -INFINITY;
  for (int64_t v = 0; v < V; ++v) {
    const float s = logit_at(row, v, dtype) / T;
    if (isnan(s)) return -1;
    if (s > m) m = s;
  }
  if (!isfinite(m)) return -1;
  double S = 0.0;
  for (int64_t v = 0; v < V; ++v) {
    const float d = logit_at(row, v, dtype) / T - m;
    S += exp((double)d);
  }
  st->m = m;
  st->lnS = log(S);
  return 0;
}

/* lp_x = fl32(s_x - m) - lnS */
static double logprob_at(const void* row, int64_t x, int dtype, float T, const row_stat* st) {
  const float d = logit_at(row, x, dtype) / T - st->m;
  return (double)d - st->lnS;
}

int svo_row_logprobs(const void* row, int64_t V, int dtype, float T, double* lp) {
  row_stat st;
  if (row_stats(row, V, dtype, T, &st) != 0) return -1;
  for (int64_t v = 0; v < V; ++v) lp[v] = logprob_at(row, v, dtype, T, &st);
  return 0;
}

/* Reading (greedy rows): at T = 0 the target is the point mass on the first
 * index of the largest raw logit. */
int64_t svo_row_argmax(const void* row, int64_t V, int dtype) {
  float best = -INFINITY;
  int64_t arg = -1;
  for (int64_t v = 0; v < V; ++v) {
    const float z = logit_at(row, v, dtype);
    if (isnan(z)) return -1;
    if (z > best) {
      best = z;
      arg = v;
    }
  }
  if (!isfinite(best)) return -1;
  return arg;
}

/* [SSD] s.2 "Saguaro sampling": the correction token is drawn from
 * r(.) proportional to max(p_target - p_draft, 0); in log space
 * log r_v = lp_v + log1p(-exp(lq_v - lp_v)) where lp_v > lq_v. */
int64_t svo_residual_logw(const double* lp, const double* lq, int64_t V, double* out) {
  int64_t n = 0;
  for (int64_t v = 0; v < V; ++v) {
    if (lp[v] > lq[v]) {
      out[v] = lp[v] + log1p(-exp(lq[v] - lp[v]));
      ++n;
    } else {
      out[v] = -INFINITY;
    }
  }
  return n;
}

/* Gumbel-max: y = argmax_v (logw_v + G_v), G_v = -ln(-ln U_v), U_v the
 * keyed Philox uniform for vocabulary entry v (counter word 0 = v >> 2, word
 * v & 3).  -ln U is evaluated as -log1p(-(1 - U)); 1 - U is exact.  Ties go
 * to the lowest v.  gap = best - second best score. */
int64_t svo_gumbel_argmax(const double* logw, int64_t V, uint64_t seed, uint64_t step,
                          uint32_t tag, uint32_t b, uint32_t pos, double* gap) {
  double best = -INFINITY, second = -INFINITY;
  int64_t arg = -1;
  for (int64_t v = 0; v < V; ++v) {
    if (logw[v] == -INFINITY) continue;
    const uint32_t x =
        svo_stream_word(seed, step, tag, b, 0, pos, (uint32_t)(v >> 2), (uint32_t)(v & 3));
    const double U = svo_u01_gumbel(x);
    const double E = -log1p(-(1.0 - U));
    const double score = logw[v] - log(E);
    if (arg < 0 || score > best) {
      second = best;
      best = score;
      arg = v;
    } else if (score > second) {
      second = score;
    }
  }
  if (gap) *gap = (arg >= 0 && second > -INFINITY) ? best - second : INFINITY;
  return arg;
}

/* Reading of the draw "from r(.)" ([SSD] s.2): any exact sampler of the
 * normalised weights qualifies; the single-draft draw takes a two-level
 * exponential race.  With W_g the summed weight of group g and E_g, E_v
 * independent unit exponentials, the group g* maximising W_g / E_g is g with
 * probability W_g / W (the minimum of independent exponential clocks of
 * rates W_g), and the entry maximising w_v / E_v within g* is v with
 * probability w_v / W_g* (the same property within the group), so v is drawn
 * with probability w_v / W.  The group noise uses its own tag, so the two
 * levels are independent.  In log space: ln W_g - ln E_g and logw_v - ln E_v. */
static double group_exponential(uint64_t seed, uint64_t step, uint32_t b, uint32_t pos,
                                int64_t g) {
  const uint32_t x = svo_stream_word(seed, step, SVO_TAG_GROUP, b, 0, pos, (uint32_t)g, 0);
  return -log1p(-(1.0 - svo_u01_gumbel(x)));
}

static double entry_exponential(uint64_t seed, uint64_t step, uint32_t tag, uint32_t b,
                                uint32_t pos, int64_t v) {
  const uint32_t x =
      svo_stream_word(seed, step, tag, b, 0, pos, (uint32_t)(v >> 2), (uint32_t)(v & 3));
  return -log1p(-(1.0 - svo_u01_gumbel(x)));
}

int64_t svo_group_race(const double* logw, int64_t V, uint64_t seed, uint64_t step,
                       uint32_t tag, uint32_t b, uint32_t pos, double* gap) {
  const int64_t G = SVO_RACE_GROUP;
  const int64_t ng = (V + G - 1) / G;
  /* level 1: the groups */
  double best = -INFINITY, second = -INFINITY;
  int64_t gbest = -1;
  for (int64_t g = 0; g < ng; ++g) {
    double W = 0.0;
    for (int64_t v = g * G; v < V && v < (g + 1) * G; ++v)
      if (logw[v] != -INFINITY) W += exp(logw[v]);
    if (!(W > 0.0)) continue;
    const double score = log(W) - log(group_exponential(seed, step, b, pos, g));
    if (gbest < 0 || score > best) {
      second = best;
      best = score;
      gbest = g;
    } else if (score > second) {
      second = score;
    }
  }
  if (gbest < 0) {
    if (gap) *gap = INFINITY;
    return -1;
  }
  const double ggap = second > -INFINITY ? best - second : INFINITY;
  /* level 2: the entries of the winning group */
  best = -INFINITY;
  second = -INFINITY;
  int64_t arg = -1;
  for (int64_t v = gbest * G; v < V && v < (gbest + 1) * G; ++v) {
    if (logw[v] == -INFINITY) continue;
    const double score = logw[v] - log(entry_exponential(seed, step, tag, b, pos, v));
    if (arg < 0 || score > best) {
      second = best;
      best = score;
      arg = v;
    } else if (score > second) {
      second = score;
    }
  }
  const double egap = second > -INFINITY ? best - second : INFINITY;
  if (gap) *gap = ggap < egap ? ggap : egap;
  return arg;
}

/* ------------------------------------------------------------------------
 * Default randomness: Philox uniforms.
 * ---------------------------------------------------------------------- */
typedef struct {
  uint64_t seed, step;
} philox_ctx;

/* Tie rule T for a single-draft draw (a reading: the pages fix no tolerance
 * for the draw).  A draw is logged as a Gumbel near-tie when another
 * candidate's score could overtake the winner's once every weight carries
 * the error of an fp32 evaluation of the probabilities: score s_v =
 * ln w_v + G_v carries u_v = GUMBEL_TIE_BAND / 2 + (eta_p p_v + eta_q q_v) /
 * w_v, with eta = 2e-6 + 2e-7 |ln prob| the relative error of a probability
 * evaluated as 2^(fp32 exponent) from temperature-scaled fp32 logits and an
 * fp32 row sum, and w_v = p_v - q_v (residual) or p_v (bonus, q = 0).  For a
 * well-conditioned weight this is the fixed band (gap < GUMBEL_TIE_BAND); a
 * residual weight of two nearly equal probabilities is ill-conditioned, and
 * its band widens by (p + q) / (p - q).  lq == NULL: bonus draw. */
static double prob_eta(double lp) { return 2e-6 + 2e-7 * fabs(lp); }

/* Group level of the same rule: an fp32 group sum lies within
 * [W_g^-, W_g^+], where each weight is moved by its evaluation error
 * d_v = eta_p p_v + eta_q q_v (and clipped at zero, so entries with p <= q
 * that rounding could make positive are counted) and the sum by its own
 * rounding (relative GROUP_SUM_ETA: a sum of non-negative fp32 terms of
 * depth at most 64).  The draw is logged when another group's score
 * ln W^+ - ln E could reach the winning group's ln W^- - ln E, each also
 * moved by half the fixed band. */
#define GROUP_SUM_ETA (64.0 * 0x1p-24)

static int draw_fragile(const double* lw, const double* lp, const double* lq, int64_t V,
                        const philox_ctx* pc, uint32_t b, uint32_t pos, int64_t y) {
  if (y < 0) return 0;
  const int64_t G = SVO_RACE_GROUP;
  const int64_t ng = (V + G - 1) / G;
  const int64_t gy = y / G;
  double lo_y = -INFINITY, hi_other = -INFINITY;
  for (int64_t g = 0; g < ng; ++g) {
    double Wlo = 0.0, Whi = 0.0;
    for (int64_t v = g * G; v < V && v < (g + 1) * G; ++v) {
      const double p = exp(lp[v]);
      const double q = lq ? exp(lq[v]) : 0.0;
      const double d = prob_eta(lp[v]) * p + (lq ? prob_eta(lq[v]) * q : 0.0);
      const double w = p - q;
      if (w - d > 0.0) Wlo += w - d;
      if (w + d > 0.0) Whi += w + d;
    }
    const double lnE = log(group_exponential(pc->seed, pc->step, b, pos, g));
    if (g == gy) {
      lo_y = Wlo > 0.0 ? log(Wlo * (1.0 - GROUP_SUM_ETA)) - lnE - 0.5 * GUMBEL_TIE_BAND : -INFINITY;
    } else if (Whi > 0.0) {
      const double hi = log(Whi * (1.0 + GROUP_SUM_ETA)) - lnE + 0.5 * GUMBEL_TIE_BAND;
      if (hi > hi_other) hi_other = hi;
    }
  }
  if (hi_other > -INFINITY && hi_other >= lo_y) return 1; /* no competitor: no group flip */
  /* entry level, within the winning group */
  double sy = -INFINITY, uy = 0.0, other = -INFINITY;
  for (int64_t v = gy * G; v < V && v < (gy + 1) * G; ++v) {
    if (lw[v] == -INFINITY) continue;
    const double E = entry_exponential(pc->seed, pc->step, SVO_TAG_GUMBEL, b, pos, v);
    const double score = lw[v] - log(E);
    const double p = exp(lp[v]);
    const double q = lq ? exp(lq[v]) : 0.0;
    const double w = exp(lw[v]);
    double u = 0.5 * GUMBEL_TIE_BAND;
    u += (prob_eta(lp[v]) * p + (lq ? prob_eta(lq[v]) * q : 0.0)) / w;
    if (v == y) {
      sy = score;
      uy = u;
    } else if (score + u > other) {
      other = score + u;
    }
  }
  return other >= sy - uy;
}

static int philox_coin(void* ctx, double h, uint32_t tag, uint32_t b, uint32_t k,
                       uint32_t pos, double* gap) {
  const philox_ctx* c = (const philox_ctx*)ctx;
  const double u = svo_u01_accept(svo_stream_word(c->seed, c->step, tag, b, k, pos, pos, 0));
  if (gap) *gap = fabs(u - h);
  return u < h;
}

static int64_t philox_categorical(void* ctx, const double* logw, int64_t V, uint32_t tag,
                                  uint32_t b, uint32_t pos, double* gap) {
  const philox_ctx* c = (const philox_ctx*)ctx;
  /* single-draft draws: the two-level race; multi-draft draws: the plain race */
  if (tag == SVO_TAG_GUMBEL) return svo_group_race(logw, V, c->seed, c->step, tag, b, pos, gap);
  return svo_gumbel_argmax(logw, V, c->seed, c->step, tag, b, pos, gap);
}

/* ------------------------------------------------------------------------
 * Single-draft verification.
 * ---------------------------------------------------------------------- */

/* [FS] s.1: a draft token is accepted when u < min(1, p/q), p/q evaluated
 * as exp(lp - lq).  Reading for q = 0: p/q = +inf if p > 0 (accept), and
 * 0/0 rejects. */
static double accept_prob(double lp, double lq) {
  if (lq == -INFINITY) return lp == -INFINITY ? 0.0 : 1.0;
  const double r = exp(lp - lq);
  return r < 1.0 ? r : 1.0;
}

static void seq_single(const char* target, const char* draft, const int32_t* tokens,
                       const float* temps, int gamma, int64_t V, int dtype, int64_t b,
                       const svo_rng* rng, const philox_ctx* pc, int32_t* out_accept_len,
                       int32_t* out_tokens,
                       double* out_lp, double* out_lq, uint8_t* out_tie) {
  const size_t es = elem_size(dtype);
  const size_t rowb = (size_t)V * es;
  const char* trow0 = target + (size_t)b * (size_t)(gamma + 1) * rowb;
  const char* drow0 = draft + (size_t)b * (size_t)gamma * rowb;
  const int32_t* x = tokens + (size_t)b * (size_t)gamma;
  int32_t* tok = out_tokens + (size_t)b * (size_t)(gamma + 1);
  uint8_t tie = 0;

  for (int i = 0; i <= gamma; ++i) tok[i] = -1;
  out_accept_len[b] = -1;
  if (out_lp)
    for (int i = 0; i < gamma; ++i) out_lp[(size_t)b * gamma + i] = NAN;
  if (out_lq)
    for (int i = 0; i < gamma; ++i) out_lq[(size_t)b * gamma + i] = NAN;
  if (out_tie) out_tie[b] = 0;

  const float T = temps[b];
  if (!(T >= 0.0f) || isinf(T)) return; /* invalid temperature */
  for (int i = 0; i < gamma; ++i)
    if (x[i] < 0 || (int64_t)x[i] >= V) return; /* token outside the vocabulary */

  if (T == 0.0f) {
    /* Greedy: accept while the draft token equals the target argmax; the
     * correction (or bonus) token is the target argmax at the stop. */
    int64_t g[MAX_STEPS + 1];
    for (int i = 0; i <= gamma; ++i) {
      g[i] = svo_row_argmax(trow0 + (size_t)i * rowb, V, dtype);
      if (g[i] < 0) return;
    }
    int j = gamma;
    for (int i = 0; i < gamma; ++i)
      if ((int64_t)x[i] != g[i]) {
        j = i;
        break;
      }
    for (int i = 0; i < j; ++i) tok[i] = x[i];
    tok[j] = (int32_t)g[j];
    out_accept_len[b] = j;
    return;
  }

  row_stat sp[MAX_STEPS + 1], sq[MAX_STEPS];
  for (int i = 0; i <= gamma; ++i)
    if (row_stats(trow0 + (size_t)i * rowb, V, dtype, T, &sp[i]) != 0) return;
  for (int i = 0; i < gamma; ++i)
    if (row_stats(drow0 + (size_t)i * rowb, V, dtype, T, &sq[i]) != 0) return;

  double lp[MAX_STEPS], lq[MAX_STEPS];
  for (int i = 0; i < gamma; ++i) {
    lp[i] = logprob_at(trow0 + (size_t)i * rowb, x[i], dtype, T, &sp[i]);
    lq[i] = logprob_at(drow0 + (size_t)i * rowb, x[i], dtype, T, &sq[i]);
  }

  /* Accept/reject in order; [FD] problem definition: the correction token is
   * drawn at the first rejection point.  Uniforms after it are never used. */
  int j = gamma;
  for (int i = 0; i < gamma; ++i) {
    double gap = INFINITY;
    const int acc = rng->coin(rng->ctx, accept_prob(lp[i], lq[i]), SVO_TAG_ACCEPT,
                              (uint32_t)b, 0, (uint32_t)i, &gap);
    if (gap < BERNOULLI_TIE_BAND) tie |= SVO_TIE_BERNOULLI;
    if (!acc) {
      j = i;
      break;
    }
  }

  double* lw = (double*)malloc((size_t)V * sizeof(double));
  double* lpr = (double*)malloc((size_t)V * sizeof(double));
  double* lqr = (double*)malloc((size_t)V * sizeof(double));
  if (!lw || !lpr || !lqr) {
    free(lw);
    free(lpr);
    free(lqr);
    return;
  }
  svo_row_logprobs(trow0 + (size_t)j * rowb, V, dtype, T, lpr);
  int residual = 0;
  if (j < gamma) {
    /* Residual max(p_j - q_j, 0).  Reading: if it is identically zero (p_j
     * == q_j to rounding), draw from p_j. */
    svo_row_logprobs(drow0 + (size_t)j * rowb, V, dtype, T, lqr);
    residual = svo_residual_logw(lpr, lqr, V, lw) != 0;
    if (!residual) memcpy(lw, lpr, (size_t)V * sizeof(double));
  } else {
    /* Every draft token accepted: bonus token from the target row gamma. */
    memcpy(lw, lpr, (size_t)V * sizeof(double));
  }
  double gap = INFINITY;
  const int64_t y = rng->categorical(rng->ctx, lw, V, SVO_TAG_GUMBEL, (uint32_t)b, (uint32_t)j, &gap);
  if (gap < GUMBEL_TIE_BAND) tie |= SVO_TIE_GUMBEL;
  if (pc && draw_fragile(lw, lpr, residual ? lqr : NULL, V, pc, (uint32_t)b, (uint32_t)j, y))
    tie |= SVO_TIE_GUMBEL;
  free(lw);
  free(lpr);
  free(lqr);

  for (int i = 0; i < j; ++i) tok[i] = x[i];
  tok[j] = (int32_t)y;
  out_accept_len[b] = j;
  if (out_lp)
    for (int i = 0; i < gamma; ++i) out_lp[(size_t)b * gamma + i] = lp[i];
  if (out_lq)
    for (int i = 0; i < gamma; ++i) out_lq[(size_t)b * gamma + i] = lq[i];
  if (out_tie) out_tie[b] = tie;
}

int svo_verify(const void* target, const void* draft, const int32_t* tokens,
               const float* temps, int64_t B, int gamma, int64_t V, int dtype,
               uint64_t seed, uint64_t step, int64_t b_begin, int64_t b_end,
               int32_t* out_accept_len, int32_t* out_tokens, double* out_lp,
               double* out_lq, uint8_t* out_tie, const svo_rng* rng) {
  if (!target || !draft || !tokens || !temps || !out_accept_len || !out_tokens) return -1;
  if (B < 0 || gamma < 1 || gamma > MAX_STEPS || V < 1 || V > ((int64_t)1 << 31)) return -1;
  if (dtype != SVO_F32 && dtype != SVO_BF16) return -1;
  if (step >> 32) return -1;
  if (b_begin < 0 || b_end > B || b_begin > b_end) return -1;
  philox_ctx pc = {seed, step};
  svo_rng def = {&pc, philox_coin, philox_categorical};
  const philox_ctx* tie_ctx = rng ? NULL : &pc; /* the draw tie rule needs the Philox stream */
  if (!rng) rng = &def;
  for (int64_t b = b_begin; b < b_end; ++b)
    seq_single((const char*)target, (const char*)draft, tokens, temps, gamma, V, dtype, b, rng,
               tie_ctx, out_accept_len, out_tokens, out_lp, out_lq, out_tie);
  return 0;
}

/* ------------------------------------------------------------------------
 * Multi-draft verification, [GBV] Algorithm 1.
 *
 * Reading (equations 2 and 4 and Algorithm 2 are not printed on the page):
 *  - Drafts are visited in index order k = 0..K-1.  A draft is considered only
 *    if its first tau tokens equal the accepted prefix.
 *  - Sub-block acceptance uses the greedy block-verification weights:
 *      w_tau = min(1, R(x_tau) / Q~(x_tau)),  w_i = min(1, w_{i-1} P_i(x_i) / Q_i(x_i)),
 *      h_i = A_i / (A_i + 1 - w_i),  A_i = sum_v max(w_i P_{i+1}(v) - Q_{i+1}(v), 0)
 *            (h_i = 1 when the denominator is 0; h_{L-1} = w_{L-1}),
 *    and the longest accepted sub-block wins (tau <- last i+1 with eta_i < h_i).
 *  - R is the current target law at position tau (P_tau at first).  On an
 *    advance, R <- norm(max(w P_tau - Q_tau, 0)) (P_L when tau reaches L) and
 *    H is cleared.  On a rejection the draft's token x_tau joins H and
 *    R <- norm(max(R - Q~, 0)).
 *  - Q~ is the draft law at position tau conditioned on not being in H
 *    (Q_tau restricted to the complement of H, renormalised).  Skipping drafts
 *    whose token is in H is only distribution-preserving with this
 *    conditioning; with the unconditioned Q_tau the output law drifts.
 *  - Finish: the correction token is drawn from R at position tau (the
 *    target row L when tau == L).
 * ---------------------------------------------------------------------- */
static double step_weight(double w, double num, double den) {
  if (den > 0.0) {
    const double t = w * (num / den);
    return t < 1.0 ? t : 1.0;
  }
  return (w > 0.0 && num > 0.0) ? 1.0 : 0.0;
}

static void seq_multi(const char* target, const char* draft, const int32_t* tokens,
                      const float* temps, int K, int L, int64_t V, int dtype, int per_draft,
                      int64_t b, const svo_rng* rng, int32_t* out_accept_len,
                      int32_t* out_tokens, int32_t* out_draft_index, uint8_t* out_tie) {
  const size_t es = elem_size(dtype);
  const size_t rowb = (size_t)V * es;
  /* Row sets: one shared by every draft, or one per draft (per_draft), in
   * which case row (k, i) is conditioned on draft k's own prefix. */
  const size_t nset = per_draft ? (size_t)K : 1u;
  const char* trow0 = target + (size_t)b * nset * (size_t)(L + 1) * rowb;
  const char* drow0 = draft + (size_t)b * nset * (size_t)L * rowb;
#define SET(k) ((size_t)(per_draft ? (k) : 0))
#define TROW(k, i) (trow0 + (SET(k) * (size_t)(L + 1) + (size_t)(i)) * rowb)
#define DROW(k, i) (drow0 + (SET(k) * (size_t)L + (size_t)(i)) * rowb)
  const int32_t* xs = tokens + (size_t)b * (size_t)K * (size_t)L;
  int32_t* tok = out_tokens + (size_t)b * (size_t)(L + 1);
  uint8_t tie = 0;

  for (int i = 0; i <= L; ++i) tok[i] = -1;
  out_accept_len[b] = -1;
  if (out_draft_index) out_draft_index[b] = -1;
  if (out_tie) out_tie[b] = 0;

  const float T = temps[b];
  if (!(T >= 0.0f) || isinf(T)) return;
  for (int64_t n = 0; n < (int64_t)K * L; ++n)
    if (xs[n] < 0 || (int64_t)xs[n] >= V) return;

  if (T == 0.0f) {
    /* Reading (greedy): the target is the argmax at every position; the
     * accepted block is the longest draft prefix that matches it (first
     * draft on ties), and the correction is the argmax at tau. */
    int64_t g[32][MAX_STEPS + 1]; /* argmax of row (set, i) */
    for (size_t k = 0; k < nset; ++k)
      for (int i = 0; i <= L; ++i) {
        g[k][i] = svo_row_argmax(TROW(k, i), V, dtype);
        if (g[k][i] < 0) return;
      }
    int tau = 0, a = -1;
    for (int k = 0; k < K; ++k) {
      int n = 0;
      while (n < L && (int64_t)xs[(size_t)k * L + n] == g[SET(k)][n]) ++n;
      if (n > tau) {
        tau = n;
        a = k;
      }
    }
    for (int i = 0; i < tau; ++i) tok[i] = xs[(size_t)a * L + i];
    /* the correction is the argmax at tau of the accepted draft's rows (every
     * draft's row 0 when nothing was accepted: they share the empty prefix) */
    tok[tau] = (int32_t)g[SET(a < 0 ? 0 : a)][tau];
    out_accept_len[b] = tau;
    if (out_draft_index) out_draft_index[b] = a;
    return;
  }

  /* Probability vectors P_0..P_L (target) and Q_0..Q_{L-1} (draft) of every
   * row set. */
  double* P = (double*)malloc(nset * (size_t)(L + 1) * (size_t)V * sizeof(double));
  double* Q = (double*)malloc(nset * (size_t)L * (size_t)V * sizeof(double));
  double* R = (double*)malloc((size_t)V * sizeof(double));
  double* lw = (double*)malloc((size_t)V * sizeof(double));
  unsigned char* inH = (unsigned char*)calloc((size_t)V, 1);
  int ok = P && Q && R && lw && inH;
  for (size_t k = 0; ok && k < nset; ++k) {
    for (int i = 0; ok && i <= L; ++i)
      ok = svo_row_logprobs(TROW(k, i), V, dtype, T, P + (k * (size_t)(L + 1) + i) * V) == 0;
    for (int i = 0; ok && i < L; ++i)
      ok = svo_row_logprobs(DROW(k, i), V, dtype, T, Q + (k * (size_t)L + i) * V) == 0;
  }
  if (!ok) goto done;
  for (size_t n = 0; n < nset * (size_t)(L + 1) * (size_t)V; ++n) P[n] = exp(P[n]);
  for (size_t n = 0; n < nset * (size_t)L * (size_t)V; ++n) Q[n] = exp(Q[n]);
  /* P_i and Q_i as seen by draft k (its own rows, or the shared ones) */
#define PROW(k, i) (P + (SET(k) * (size_t)(L + 1) + (size_t)(i)) * (size_t)V)
#define QROW(k, i) (Q + (SET(k) * (size_t)L + (size_t)(i)) * (size_t)V)

  int tau = 0, a = -1;
  double qH = 0.0; /* Q_tau mass of H */
  memcpy(R, PROW(0, 0), (size_t)V * sizeof(double)); /* every draft shares the empty prefix */

  for (int k = 0; k < K; ++k) {
    if (tau == L) break;
    const int32_t* x = xs + (size_t)k * L;
    if (tau > 0 && memcmp(x, xs + (size_t)a * L, (size_t)tau * sizeof(int32_t)) != 0) continue;
    if (inH[x[tau]]) continue; /* rejected sub-block seen before */

    const double keep = 1.0 - qH;
    const double qfirst = keep > 0.0 ? QROW(k, tau)[x[tau]] / keep : 0.0;
    double w = 1.0, wbest = 1.0;
    int best = tau;
    for (int i = tau; i < L; ++i) {
      if (i == tau)
        w = step_weight(w, R[x[i]], qfirst);
      else
        w = step_weight(w, PROW(k, i)[x[i]], QROW(k, i)[x[i]]);
      double h;
      if (i < L - 1) {
        double A = 0.0;
        const double* pn = PROW(k, i + 1);
        const double* qn = QROW(k, i + 1);
        for (int64_t v = 0; v < V; ++v) {
          const double t = w * pn[v] - qn[v];
          if (t > 0.0) A += t;
        }
        const double den = A + 1.0 - w;
        h = den == 0.0 ? 1.0 : A / den;
      } else {
        h = w;
      }
      double gap = INFINITY;
      if (rng->coin(rng->ctx, h, SVO_TAG_MD_ETA, (uint32_t)b, (uint32_t)k, (uint32_t)i, &gap)) {
        best = i + 1;
        wbest = w;
      }
      if (gap < BERNOULLI_TIE_BAND) tie |= SVO_TIE_BERNOULLI;
    }

    if (best > tau) {
      tau = best;
      a = k;
      memset(inH, 0, (size_t)V);
      qH = 0.0;
      if (tau < L) {
        double Z = 0.0;
        for (int64_t v = 0; v < V; ++v) {
          const double t = wbest * PROW(k, tau)[v] - QROW(k, tau)[v];
          R[v] = t > 0.0 ? t : 0.0;
          Z += R[v];
        }
        if (Z > 0.0)
          for (int64_t v = 0; v < V; ++v) R[v] /= Z;
        else
          memcpy(R, PROW(k, tau), (size_t)V * sizeof(double));
      }
    } else {
      double Z = 0.0;
      for (int64_t v = 0; v < V; ++v) {
        const double qt = (inH[v] || keep <= 0.0) ? 0.0 : QROW(k, tau)[v] / keep;
        const double t = R[v] - qt;
        lw[v] = t > 0.0 ? t : 0.0;
        Z += lw[v];
      }
      if (Z > 0.0)
        for (int64_t v = 0; v < V; ++v) R[v] = lw[v] / Z;
      inH[x[tau]] = 1;
      qH += QROW(k, tau)[x[tau]];
    }
  }

  /* [GBV] termination: whole block accepted -> correction from the target
   * (row L); otherwise from the residual law R at tau. */
  if (tau == L) {
    for (int64_t v = 0; v < V; ++v) lw[v] = log(PROW(a, L)[v]);
  } else {
    for (int64_t v = 0; v < V; ++v) lw[v] = R[v] > 0.0 ? log(R[v]) : -INFINITY;
  }
  {
    double gap = INFINITY;
    const int64_t y =
        rng->categorical(rng->ctx, lw, V, SVO_TAG_MD_GUMBEL, (uint32_t)b, (uint32_t)tau, &gap);
    if (gap < GUMBEL_TIE_BAND) tie |= SVO_TIE_GUMBEL;
    for (int i = 0; i < tau; ++i) tok[i] = xs[(size_t)a * L + i];
    tok[tau] = (int32_t)y;
    out_accept_len[b] = tau;
    if (out_draft_index) out_draft_index[b] = a;
    if (out_tie) out_tie[b] = tie;
  }
#undef PROW
#undef QROW
#undef TROW
#undef DROW
#undef SET
done:
  free(P);
  free(Q);
  free(R);
  free(lw);
  free(inH);
}

int svo_verify_multidraft(const void* target, const void* draft, const int32_t* tokens,
                          const float* temps, int64_t B, int K, int L, int64_t V,
                          int dtype, uint64_t seed, uint64_t step, int64_t b_begin,
                          int64_t b_end, int32_t* out_accept_len, int32_t* out_tokens,
                          int32_t* out_draft_index, uint8_t* out_tie, const svo_rng* rng) {
  return svo_verify_multidraft_rows(target, draft, tokens, temps, B, K, L, V, dtype, 0, seed,
                                    step, b_begin, b_end, out_accept_len, out_tokens,
                                    out_draft_index, out_tie, rng);
}

int svo_verify_multidraft_rows(const void* target, const void* draft, const int32_t* tokens,
                               const float* temps, int64_t B, int K, int L, int64_t V,
                               int dtype, int per_draft, uint64_t seed, uint64_t step,
                               int64_t b_begin, int64_t b_end, int32_t* out_accept_len,
                               int32_t* out_tokens, int32_t* out_draft_index,
                               uint8_t* out_tie, const svo_rng* rng) {
  if (!target || !draft || !tokens || !temps || !out_accept_len || !out_tokens) return -1;
  if (B < 0 || K < 1 || K > 32 || L < 1 || L > MAX_STEPS || V < 1 || V > ((int64_t)1 << 31))
    return -1;
  if (dtype != SVO_F32 && dtype != SVO_BF16) return -1;
  if (step >> 32) return -1;
  if (b_begin < 0 || b_end > B || b_begin > b_end) return -1;
  philox_ctx pc = {seed, step};
  svo_rng def = {&pc, philox_coin, philox_categorical};
  if (!rng) rng = &def;
  for (int64_t b = b_begin; b < b_end; ++b)
    seq_multi((const char*)target, (const char*)draft, tokens, temps, K, L, V, dtype,
              per_draft != 0, b, rng, out_accept_len, out_tokens, out_draft_index, out_tie);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Draft selection as a K-armed bandit ([FS] Methodology s.2): before each
 * decoding step one draft model (an arm) is chosen from the acceptance
 * history alone; the reward of a step is its fraction of accepted draft
 * tokens, in [0, 1].  Two policies, as the page lists them:
 *  - UCB1 (Auer, Cesa-Bianchi, Fischer, "Finite-time Analysis of the
 *    Multiarmed Bandit Problem", 2002): every arm once, in index order; then
 *    the arm with the largest mean reward + sqrt(2 ln n / n_j), n the number
 *    of pulls so far; ties go to the lower index.
 *  - Thompson Sampling for rewards in [0, 1] (Agrawal, Goyal, "Analysis of
 *    Thompson Sampling for the Multi-armed Bandit Problem", 2012): a
 *    Beta(S_j + 1, F_j + 1) draw per arm, the largest draw wins (ties to the
 *    lower index); a reward r counts as a success with probability r (one
 *    Bernoulli trial), else as a failure.
 * Randomness: Philox4x32-10 keyed by the seed; counter (c0, round, slot,
 * tag << 24) with tag 5 for the Beta draws (slot = 2 arm + {0: X, 1: Y} of
 * Beta = X / (X + Y) with X, Y Gamma) and tag 6 for the success trials
 * (slot = arm).  A uniform in (0, 1) takes two words w0, w1 of a block:
 * m = ((w0 << 32) | w1) >> 12, u = (2m + 1) 2^-53, exact in fp64.
 * Gamma(alpha >= 1) by Marsaglia and Tsang ("A Simple Method for Generating
 * Gamma Variables", 2000): d = alpha - 1/3, c = 1 / sqrt(9 d); repeat
 * z ~ N(0, 1), v = (1 + c z)^3 while v <= 0 or
 * ln u >= z^2 / 2 + d - d v + d ln v; return d v.  Iteration i takes u1, u2
 * from Philox block c0 = i (word pairs 0-1 and 2-3), z = sqrt(-2 ln u1)
 * cos(2 pi u2) (Box-Muller), and u from block c0 = i + 2^31 (words 0-1).  At
 * most 64 iterations (then d is returned; each is accepted with probability
 * above 0.95).
 * ------------------------------------------------------------------------ */
#define BANDIT_TAG_BETA 5u
#define BANDIT_TAG_TRIAL 6u
#define GAMMA_MAX_ITERS 64
#define TWO_PI 6.283185307179586476925 /* 2 pi, rounded to the nearest double */

static double u01_pair(uint32_t w0, uint32_t w1) {
  const uint64_t m = ((((uint64_t)w0) << 32) | (uint64_t)w1) >> 12;
  return (double)(2u * m + 1u) * 0x1p-53;
}

static void bandit_block(uint64_t seed, uint32_t c0, uint32_t round, uint32_t slot, uint32_t tag,
                         uint32_t out[4]) {
  const uint32_t ctr[4] = {c0, round, slot, tag << 24};
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  svo_philox4x32_10(ctr, key, out);
}

double svo_bandit_uniform(uint64_t seed, uint32_t c0, uint32_t round, uint32_t slot, uint32_t tag,
                          int half) {
  uint32_t w[4];
  bandit_block(seed, c0, round, slot, tag, w);
  return half ? u01_pair(w[2], w[3]) : u01_pair(w[0], w[1]);
}

double svo_gamma_sample(double alpha, uint64_t seed, uint32_t round, uint32_t slot) {
  if (!(alpha >= 1.0)) return NAN;
  const double d = alpha - 1.0 / 3.0;
  const double c = 1.0 / sqrt(9.0 * d);
  for (uint32_t i = 0; i < GAMMA_MAX_ITERS; ++i) {
    uint32_t w[4], w3[4];
    bandit_block(seed, i, round, slot, BANDIT_TAG_BETA, w);
    bandit_block(seed, i + 0x80000000u, round, slot, BANDIT_TAG_BETA, w3);
    const double u1 = u01_pair(w[0], w[1]);
    const double u2 = u01_pair(w[2], w[3]);
    const double u = u01_pair(w3[0], w3[1]);
    const double z = sqrt(-2.0 * log(u1)) * cos(TWO_PI * u2);
    const double t = 1.0 + c * z;
    if (t <= 0.0) continue;
    const double v = t * t * t;
    if (log(u) < 0.5 * z * z + d - d * v + d * log(v)) return d * v;
  }
  return d;
}

double svo_beta_sample(double a, double b, uint64_t seed, uint32_t round, uint32_t arm) {
  const double x = svo_gamma_sample(a, seed, round, 2u * arm);
  const double y = svo_gamma_sample(b, seed, round, 2u * arm + 1u);
  return x / (x + y);
}

int svo_ucb1_select(int K, const int64_t* pulls, const double* reward_sum) {
  if (K < 1 || !pulls || !reward_sum) return -1;
  int64_t n = 0;
  for (int j = 0; j < K; ++j) {
    if (pulls[j] == 0) return j; /* every arm once, in index order */
    n += pulls[j];
  }
  int best = 0;
  double best_v = -INFINITY;
  for (int j = 0; j < K; ++j) {
    const double mean = reward_sum[j] / (double)pulls[j];
    const double v = mean + sqrt(2.0 * log((double)n) / (double)pulls[j]);
    if (v > best_v) {
      best_v = v;
      best = j;
    }
  }
  return best;
}

int svo_thompson_select(int K, const int64_t* succ, const int64_t* fail, uint64_t seed,
                        uint32_t round, double* theta) {
  if (K < 1 || !succ || !fail) return -1;
  int best = 0;
  double best_v = -INFINITY;
  for (int j = 0; j < K; ++j) {
    const double t = svo_beta_sample((double)succ[j] + 1.0, (double)fail[j] + 1.0, seed, round,
                                     (uint32_t)j);
    if (theta) theta[j] = t;
    if (t > best_v) {
      best_v = t;
      best = j;
    }
  }
  return best;
}

int svo_thompson_trial(double reward, uint64_t seed, uint32_t round, uint32_t arm) {
  return svo_bandit_uniform(seed, 0u, round, arm, BANDIT_TAG_TRIAL, 0) < reward ? 1 : 0;
}
