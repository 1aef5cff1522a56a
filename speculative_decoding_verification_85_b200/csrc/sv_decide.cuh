// sv_decide.cuh -- the single-draft decision of one sequence, taken by one
// warp from the sequence's merged row statistics (FlashSpec, Methodology s.1:
// log-space acceptance test on device; FlexDraft, Problem definition: the
// first rejection point).
#pragma once

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace sv {

// Acceptance probability min(1, p/q) from log-probabilities (fp64); q = 0
// accepts when p > 0, 0/0 rejects.
__device__ __forceinline__ double accept_prob(double lp, double lq) {
  if (lq == -INFINITY) return lp == -INFINITY ? 0.0 : 1.0;
  const double r = exp(lp - lq);
  return r < 1.0 ? r : 1.0;
}

// One warp: validate, accept/reject and (if `outputs`) write the outputs.
// T is sequence b's temperature, x[0..gamma) its draft tokens (in shared
// memory), rows[] its merged row statistics (target rows 0..gamma, then the
// draft rows), zsel[2i], zsel[2i + 1] the draft token's target / draft logit
// (or NULL: read from the rows in global memory), upre[i] the acceptance
// uniform of position i if already drawn (or NULL: drawn here).  Lane 0
// writes the hand-off record for the draw to *dst (global or shared memory).
template <bool kBf16>
__device__ __noinline__ void decide_single(const CallParams& p, int b, float T, const int* x,
                                           const RowAcc* rows, const float* zsel, SeqInfo* dst,
                                           bool outputs, const float* upre) {
  const int lane = threadIdx.x & 31;
  const int g = p.gamma;
  const bool tvalid = (T >= 0.0f) && !isinf(T);
  int32_t* tok = p.out_tokens + static_cast<size_t>(b) * (g + 1);

  bool ok = tvalid;
  int xi[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    if (i < g) {
      xi[h] = x[i];
      ok = ok && xi[h] >= 0 && xi[h] < p.V;
    }
  }
  if (tvalid) {
    const bool greedy = (T == 0.0f);
    for (int r = lane; r < p.rps; r += 32) {
      const bool needed = !greedy || r <= g;
      if (needed) {
        const RowAcc& a = rows[r];
        bool rv = !a.bad && isfinite(a.m);
        if (!greedy) rv = rv && isfinite(__fdiv_rn(a.m, T));
        ok = ok && rv;
      }
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) {
    if (outputs) {
      for (int i = lane; i <= g; i += 32) tok[i] = -1;
      for (int i = lane; i < g; i += 32) {
        if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
        if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
      }
    }
    if (lane == 0) {
      if (outputs) p.accept_len[b] = -1;
      SeqInfo si{};
      si.mode = kModeNone;
      si.j = -1;
      *dst = si;
    }
    return;
  }

  unsigned rej[2];
  if (T == 0.0f) {
    // Greedy: accept while the draft token is the first argmax of the raw row.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = lane + 32 * h;
      rej[h] = __ballot_sync(0xffffffffu, i < g && xi[h] != rows[i].arg);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = lane + 32 * h;
      bool reject = false;
      if (i < g) {
        constexpr size_t es = kBf16 ? 2 : 4;
        const char* tr = static_cast<const char*>(p.target) +
                         (static_cast<size_t>(b) * (g + 1) + i) * static_cast<size_t>(p.V) * es;
        const char* dr = static_cast<const char*>(p.draft) +
                         (static_cast<size_t>(b) * g + i) * static_cast<size_t>(p.V) * es;
        const RowAcc& ap = rows[i];
        const RowAcc& aq = rows[g + 1 + i];
        // d = fl32(fl32(z_x / T) - fl32(zmax / T)): the same fp32 operations
        // as scaling the whole row and shifting by its maximum.
        // the draft token's logits were picked up while the rows streamed
        const float zp = zsel ? zsel[2 * i] : logit_at<kBf16>(tr, xi[h]);
        const float zq = zsel ? zsel[2 * i + 1] : logit_at<kBf16>(dr, xi[h]);
        const float dp = __fsub_rn(__fdiv_rn(zp, T), __fdiv_rn(ap.m, T));
        const float dq = __fsub_rn(__fdiv_rn(zq, T), __fdiv_rn(aq.m, T));
        const double lp = static_cast<double>(dp) - log(static_cast<double>(ap.s));
        const double lq = static_cast<double>(dq) - log(static_cast<double>(aq.s));
        const double u = upre ? static_cast<double>(upre[i])
                              : accept_uniform(keyed_block(p.seed, p.step, kTagAccept, b, 0, i, i).x);
        reject = !(u < accept_prob(lp, lq));
        if (outputs && p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = static_cast<float>(lp);
        if (outputs && p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = static_cast<float>(lq);
      }
      rej[h] = __ballot_sync(0xffffffffu, reject);
    }
  }
  const int j = rej[0] ? __ffs(rej[0]) - 1 : (rej[1] ? 32 + __ffs(rej[1]) - 1 : g);

  if (outputs) for (int i = lane; i <= g; i += 32) tok[i] = i < j ? x[i] : -1;
  if (outputs && T == 0.0f) {
    for (int i = lane; i < g; i += 32) {
      if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
      if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
    }
  }
  __syncwarp();
  if (lane == 0) {
    if (outputs) p.accept_len[b] = j;
    SeqInfo si{};
    si.j = j;
    if (T == 0.0f) {
      if (outputs) tok[j] = rows[j].arg;
      si.mode = kModeNone;
    } else {
      const float c = __fdiv_rn(kLog2e, T);
      si.mode = j < g ? kModeResidual : kModeBonus;
      si.j = j;
      si.c = c;
      si.zmp = rows[j].m;
      si.lsp = log2f(rows[j].s);
      if (j < g) {
        si.zmq = rows[g + 1 + j].m;
        si.lsq = log2f(rows[g + 1 + j].s);
      }
    }
    *dst = si;
  }
}

}  // namespace sv
