// sv_bandit.cpp -- online draft selection (the host side of the library).
//
// "FlashSpec: Adaptive Speculative Decoding with Online Bandit Draft
// Selection and Triton-Optimised Verification", Methodology s.2: before each
// decoding step a draft model (an arm) is chosen from the acceptance history
// alone; the reward of a step is its fraction of accepted draft tokens.  The
// policies and the random streams are specified in include/sv_bandit.h.
//
// Philox4x32-10 here is a host implementation of Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11); Gamma variates follow
// Marsaglia and Tsang, "A Simple Method for Generating Gamma Variables"
// (2000), with Box-Muller normals.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <new>
#include <vector>

#include "spec_verify.h"
#include "sv_bandit.h"
#include "sv_internal.h"

namespace {

constexpr uint32_t kTagBeta = 5;
constexpr uint32_t kTagTrial = 6;
constexpr int kGammaIterations = 64;  // Marsaglia-Tsang accepts each try w.p. > 0.95
constexpr double kTwoPi = 6.283185307179586476925;

struct Block {
  uint32_t w[4];
};

// Philox4x32-10: ten rounds of two 32 x 32 -> 64-bit products (of words 0
// and 2) whose high halves are xored into the other words with the round
// key; the key advances by the Weyl increments between rounds.
Block philox(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint64_t seed) {
  uint32_t x0 = c0, x1 = c1, x2 = c2, x3 = c3;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    const uint64_t a = static_cast<uint64_t>(x0) * 0xD2511F53u;
    const uint64_t b = static_cast<uint64_t>(x2) * 0xCD9E8D57u;
    const uint32_t y0 = static_cast<uint32_t>(b >> 32) ^ x1 ^ k0;
    const uint32_t y2 = static_cast<uint32_t>(a >> 32) ^ x3 ^ k1;
    x1 = static_cast<uint32_t>(b);
    x3 = static_cast<uint32_t>(a);
    x0 = y0;
    x2 = y2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return Block{{x0, x1, x2, x3}};
}

// (2m + 1) 2^-53 for the top 52 bits m of (hi, lo): a double in (0, 1).
double open_unit(uint32_t hi, uint32_t lo) {
  const uint64_t m = ((static_cast<uint64_t>(hi) << 32) | lo) >> 12;
  return static_cast<double>(2 * m + 1) * 0x1p-53;
}

// Gamma(shape, 1) for shape >= 1, from the stream (round, slot, tag 5):
// try i reads u1, u2 from block c0 = i and u from block c0 = i + 2^31.
double gamma_variate(double shape, uint64_t seed, uint32_t round, uint32_t slot) {
  const double d = shape - 1.0 / 3.0;
  const double c = 1.0 / std::sqrt(9.0 * d);
  for (uint32_t i = 0; i < static_cast<uint32_t>(kGammaIterations); ++i) {
    const Block p = philox(i, round, slot, kTagBeta << 24, seed);
    const Block q = philox(i + 0x80000000u, round, slot, kTagBeta << 24, seed);
    const double u1 = open_unit(p.w[0], p.w[1]);
    const double u2 = open_unit(p.w[2], p.w[3]);
    const double u = open_unit(q.w[0], q.w[1]);
    const double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(kTwoPi * u2);
    const double t = 1.0 + c * z;
    if (t <= 0.0) continue;
    const double v = t * t * t;
    if (std::log(u) < 0.5 * z * z + d - d * v + d * std::log(v)) return d * v;
  }
  return d;
}

}  // namespace

struct sv_bandit {
  int K;
  int policy;
  uint64_t seed;
  uint32_t select_round = 0;
  uint32_t update_round = 0;
  std::vector<int64_t> pulls, succ, fail;
  std::vector<double> sums;
  std::mutex mu;
};

namespace {

int choose_ucb1(const sv_bandit& h) {
  int64_t n = 0;
  for (int j = 0; j < h.K; ++j) {
    if (h.pulls[j] == 0) return j;  // every arm once, in index order
    n += h.pulls[j];
  }
  const double log_n = std::log(static_cast<double>(n));
  int best = 0;
  double best_v = -INFINITY;
  for (int j = 0; j < h.K; ++j) {
    const double mean = h.sums[j] / static_cast<double>(h.pulls[j]);
    const double v = mean + std::sqrt(2.0 * log_n / static_cast<double>(h.pulls[j]));
    if (v > best_v) {  // strict: ties keep the lower index
      best_v = v;
      best = j;
    }
  }
  return best;
}

int choose_thompson(const sv_bandit& h) {
  int best = 0;
  double best_v = -INFINITY;
  for (int j = 0; j < h.K; ++j) {
    const uint32_t slot = 2u * static_cast<uint32_t>(j);
    const double x = gamma_variate(static_cast<double>(h.succ[j]) + 1.0, h.seed, h.select_round, slot);
    const double y = gamma_variate(static_cast<double>(h.fail[j]) + 1.0, h.seed, h.select_round, slot + 1);
    const double theta = x / (x + y);
    if (theta > best_v) {
      best_v = theta;
      best = j;
    }
  }
  return best;
}

int record(sv_bandit* h, int arm, double reward) {
  h->pulls[arm] += 1;
  h->sums[arm] += reward;
  if (h->policy == SV_BANDIT_THOMPSON) {
    const Block p = philox(0u, h->update_round, static_cast<uint32_t>(arm), kTagTrial << 24, h->seed);
    if (open_unit(p.w[0], p.w[1]) < reward)
      h->succ[arm] += 1;
    else
      h->fail[arm] += 1;
  }
  h->update_round += 1;
  return SV_OK;
}

}  // namespace

extern "C" {

sv_bandit* sv_bandit_create(int K, int policy, uint64_t seed) {
  if (K < 1 || K > SV_BANDIT_MAX_ARMS) {
    sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_create: K must be in [1, %d] (got %d)",
                  SV_BANDIT_MAX_ARMS, K);
    return nullptr;
  }
  if (policy != SV_BANDIT_UCB1 && policy != SV_BANDIT_THOMPSON) {
    sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_create: unknown policy %d", policy);
    return nullptr;
  }
  sv_bandit* h = new (std::nothrow) sv_bandit();
  if (!h) {
    sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_create: out of host memory");
    return nullptr;
  }
  h->K = K;
  h->policy = policy;
  h->seed = seed;
  h->pulls.assign(K, 0);
  h->succ.assign(K, 0);
  h->fail.assign(K, 0);
  h->sums.assign(K, 0.0);
  return h;
}

void sv_bandit_destroy(sv_bandit* h) { delete h; }

int sv_bandit_select(sv_bandit* h, int* out_arm) {
  if (!h || !out_arm) return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_select: NULL argument");
  std::lock_guard<std::mutex> lk(h->mu);
  *out_arm = h->policy == SV_BANDIT_UCB1 ? choose_ucb1(*h) : choose_thompson(*h);
  h->select_round += 1;
  return SV_OK;
}

int sv_bandit_update(sv_bandit* h, int arm, double reward) {
  if (!h) return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update: NULL handle");
  if (arm < 0 || arm >= h->K)
    return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update: arm %d not in [0, %d)", arm, h->K);
  if (!(reward >= 0.0 && reward <= 1.0))
    return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update: reward must be in [0, 1]");
  std::lock_guard<std::mutex> lk(h->mu);
  return record(h, arm, reward);
}

int sv_bandit_update_accept(sv_bandit* h, int arm, const int32_t* accept_len, int B, int gamma) {
  if (!h) return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update_accept: NULL handle");
  if (arm < 0 || arm >= h->K)
    return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update_accept: arm %d not in [0, %d)", arm,
                         h->K);
  if (B < 0 || gamma < 1 || (B > 0 && !accept_len))
    return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update_accept: bad B, gamma or pointer");
  double sum = 0.0;
  int64_t valid = 0;
  for (int b = 0; b < B; ++b) {
    const int32_t a = accept_len[b];
    if (a < 0) continue;  // an invalid sequence carries no information
    if (a > gamma)
      return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_update_accept: accept_len %d > gamma %d",
                           a, gamma);
    sum += static_cast<double>(a) / static_cast<double>(gamma);
    ++valid;
  }
  if (valid == 0) return SV_OK;
  std::lock_guard<std::mutex> lk(h->mu);
  return record(h, arm, sum / static_cast<double>(valid));
}

int sv_bandit_stats(sv_bandit* h, int64_t* pulls, double* reward_sum) {
  if (!h) return sv::set_error(SV_ERR_INVALID_ARG, "sv_bandit_stats: NULL handle");
  std::lock_guard<std::mutex> lk(h->mu);
  for (int j = 0; j < h->K; ++j) {
    if (pulls) pulls[j] = h->pulls[j];
    if (reward_sum) reward_sum[j] = h->sums[j];
  }
  return SV_OK;
}

}  // extern "C"
