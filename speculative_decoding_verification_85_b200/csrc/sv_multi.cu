// sv_multi.cu -- multi-draft verification, "SpecTr-GBV: Multi-Draft Block
// Verification Accelerating Speculative Decoding", Methodology, Algorithm 1.
//
// Pass 1 is the single-draft row pass (sv_rows.cuh) over the L+1 target and
// L draft rows of each sequence; its last CTA per sequence publishes the
// combined row statistics.  The sequential part -- drafts visited in order,
// sub-block weights w, acceptance h = A / (A + 1 - w) with
// A = sum_v max(w P_{i+1}(v) - Q_{i+1}(v), 0), the residual law R at tau and
// the rejected set H -- runs in one CTA per sequence; every V-wide quantity
// (A, the residual update, the final race) is a block reduction.
//
// Reading of the unprinted equations (as in the CPU definition): greedy
// block-verification weights; the longest accepted sub-block wins; on a
// rejection the draft law at tau is conditioned on not being in H and
// R <- norm(max(R - Q~, 0)); on an advance R <- norm(max(w P_tau - Q_tau, 0)).
// A token in H has R = 0 after its rejection, so the residual update needs
// no membership test; H only decides which later drafts are skipped.
#include <climits>

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace sv {

template <bool kBf16>
__global__ void __launch_bounds__(kP1Threads) pass1_multi_kernel(Pass1Params p) {
  __shared__ RowAcc rows[kMaxRowsPerSeq];
  const int item = blockIdx.x;
  const int rowg = item / p.nc;
  const int chunk = item - rowg * p.nc;
  const int b = rowg / p.rps;
  const int r = rowg - b * p.rps;
  if (!pass1_chunk<kBf16>(p, b, r, chunk)) return;
  combine_rows<kP1Threads>(p, b, rows);
  for (int q = threadIdx.x; q < p.rps; q += kP1Threads)
    store_partial(p.rowstat + static_cast<size_t>(b) * p.rps + q, rows[q]);
}

__device__ __forceinline__ double step_weight(double w, double num, double den) {
  if (den > 0.0) {
    const double t = w * (num / den);
    return t < 1.0 ? t : 1.0;
  }
  return (w > 0.0 && num > 0.0) ? 1.0 : 0.0;
}

template <bool kBf16>
__global__ void __launch_bounds__(kMdThreads) md_gbv_kernel(MdParams p) {
  constexpr size_t es = kBf16 ? 2 : 4;
  __shared__ float s_mt[kMaxRowsPerSeq];  // raw row maximum m
  __shared__ float s_is[kMaxRowsPerSeq];  // 1 / s, s = sum_v 2^{(z_v - m) c}
  __shared__ int s_arg[kMaxRowsPerSeq];
  __shared__ int s_x[SV_MAX_DRAFTS * SV_MAX_GAMMA];
  __shared__ int s_H[SV_MAX_DRAFTS];
  __shared__ double s_red[33];
  __shared__ float4 s_race[kMdThreads / 32];
  __shared__ int s_tau, s_a, s_nH, s_skip, s_best;
  __shared__ double s_qH, s_Rn, s_w, s_wbest, s_keep, s_qfirst;

  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int K = p.K, L = p.L, V = p.V, rps = 2 * L + 1;
  const float T = __ldg(p.temps + b);
  const char* tgt = static_cast<const char*>(p.target) +
                    static_cast<size_t>(b) * (L + 1) * static_cast<size_t>(V) * es;
  const char* drf = static_cast<const char*>(p.draft) +
                    static_cast<size_t>(b) * L * static_cast<size_t>(V) * es;
  const size_t rowb = static_cast<size_t>(V) * es;
  float* R = p.R + static_cast<size_t>(b) * V;
  int32_t* tok = p.out_tokens + static_cast<size_t>(b) * (L + 1);

  const bool tvalid = (T >= 0.0f) && !isinf(T);
  const bool greedy = tvalid && T == 0.0f;
  bool ok = tvalid;
  for (int r = tid; r < rps; r += kMdThreads) {
    const RowAcc a = load_partial(p.rowstat + static_cast<size_t>(b) * rps + r);
    s_arg[r] = a.arg;
    s_mt[r] = 0.0f;
    s_is[r] = 0.0f;
    const bool needed = tvalid && (!greedy || r <= L);
    if (needed) {
      bool rv = !a.bad && isfinite(a.m);
      if (!greedy) {
        s_mt[r] = a.m;
        s_is[r] = 1.0f / a.s;
        rv = rv && isfinite(__fdiv_rn(a.m, T));
      }
      ok = ok && rv;
    }
  }
  for (int n = tid; n < K * L; n += kMdThreads) {
    const int xv = __ldg(p.tokens + static_cast<size_t>(b) * K * L + n);
    s_x[n] = xv;
    ok = ok && xv >= 0 && xv < V;
  }
  ok = __syncthreads_and(ok);
  if (!ok) {
    for (int i = tid; i <= L; i += kMdThreads) tok[i] = -1;
    if (tid == 0) {
      p.accept_len[b] = -1;
      if (p.out_draft_index) p.out_draft_index[b] = -1;
    }
    return;
  }

  if (greedy) {
    if (tid == 0) {
      int tau = 0, a = -1;
      for (int k = 0; k < K; ++k) {
        int n = 0;
        while (n < L && s_x[k * L + n] == s_arg[n]) ++n;
        if (n > tau) {
          tau = n;
          a = k;
        }
      }
      for (int i = 0; i <= L; ++i) tok[i] = i < tau ? s_x[a * L + i] : (i == tau ? s_arg[tau] : -1);
      p.accept_len[b] = tau;
      if (p.out_draft_index) p.out_draft_index[b] = a;
    }
    return;
  }

  // P_r(v) and Q_r(v): p = 2^{(z - m) c} / s with c = log2(e) / T, the same
  // MUFU exponential that built the row sums s (so each law sums to 1 to
  // within the exponential's 2^-22 relative error), one subtraction, one
  // multiply, one ex2 and one multiply per value.
  const float cc = __fdiv_rn(kLog2e, T);
  auto prob_t = [&](int r, int v) -> float {
    return ex2_approx((logit_at<kBf16>(tgt + r * rowb, v) - s_mt[r]) * cc) * s_is[r];
  };
  auto prob_d = [&](int r, int v) -> float {
    return ex2_approx((logit_at<kBf16>(drf + r * rowb, v) - s_mt[L + 1 + r]) * cc) * s_is[L + 1 + r];
  };

  // R <- P_0
  {
    double loc = 0.0;
    for (int v = tid; v < V; v += kMdThreads) {
      const float pv = prob_t(0, v);
      R[v] = pv;
      loc += pv;
    }
    const double tot = block_sum<kMdThreads>(loc, s_red);
    if (tid == 0) {
      s_Rn = tot;
      s_tau = 0;
      s_a = -1;
      s_nH = 0;
      s_qH = 0.0;
    }
  }
  __syncthreads();

  for (int k = 0; k < K; ++k) {
    __syncthreads();  // every thread is done with the previous draft's shared state
    if (tid == 0) {
      const int tau = s_tau;
      int skip = tau == L ? 2 : 0;
      const int* x = s_x + k * L;
      if (!skip && tau > 0) {
        const int* xa = s_x + s_a * L;
        for (int i = 0; i < tau; ++i)
          if (x[i] != xa[i]) skip = 1;
      }
      if (!skip)
        for (int h = 0; h < s_nH; ++h)
          if (s_H[h] == x[tau]) skip = 1;
      s_skip = skip;
      if (!skip) {
        const double keep = 1.0 - s_qH;
        s_keep = keep;
        s_qfirst = keep > 0.0 ? static_cast<double>(prob_d(tau, x[tau])) / keep : 0.0;
        s_w = 1.0;
        s_wbest = 1.0;
        s_best = tau;
      }
    }
    __syncthreads();
    if (s_skip == 2) break;
    if (s_skip) continue;
    const int tau = s_tau;
    const int* x = s_x + k * L;
    for (int i = tau; i < L; ++i) {
      if (tid == 0) {
        double num, den;
        if (i == tau) {
          num = static_cast<double>(R[x[i]]) / s_Rn;
          den = s_qfirst;
        } else {
          num = prob_t(i, x[i]);
          den = prob_d(i, x[i]);
        }
        s_w = step_weight(s_w, num, den);
      }
      __syncthreads();
      const double w = s_w;
      double h;
      if (i < L - 1) {
        const float wf = static_cast<float>(w);
        double loc = 0.0;
        for (int v = tid; v < V; v += kMdThreads) {
          const float t = wf * prob_t(i + 1, v) - prob_d(i + 1, v);
          if (t > 0.0f) loc += t;
        }
        const double A = block_sum<kMdThreads>(loc, s_red);
        const double den = A + 1.0 - w;
        h = den == 0.0 ? 1.0 : A / den;
      } else {
        h = w;
      }
      if (tid == 0) {
        const uint4 rnd = keyed_block(p.seed, p.step, kTagMdEta, b, k, i, i);
        if (accept_uniform(rnd.x) < h) {
          s_best = i + 1;
          s_wbest = w;
        }
      }
      __syncthreads();
    }
    const int best = s_best;
    __syncthreads();
    if (best > tau) {
      if (best < L) {
        const float wb = static_cast<float>(s_wbest);
        double loc = 0.0;
        for (int v = tid; v < V; v += kMdThreads) {
          const float t = wb * prob_t(best, v) - prob_d(best, v);
          const float rv = t > 0.0f ? t : 0.0f;
          R[v] = rv;
          loc += rv;
        }
        const double tot = block_sum<kMdThreads>(loc, s_red);
        if (tid == 0) s_Rn = tot;
      }
      if (tid == 0) {
        s_tau = best;
        s_a = k;
        s_nH = 0;
        s_qH = 0.0;
      }
    } else {
      const float inv_rn = static_cast<float>(1.0 / s_Rn);
      const double keep = s_keep;
      const float inv_keep = keep > 0.0 ? static_cast<float>(1.0 / keep) : 0.0f;
      double loc = 0.0;
      for (int v = tid; v < V; v += kMdThreads) {
        const float t = R[v] * inv_rn - prob_d(tau, v) * inv_keep;
        const float rv = t > 0.0f ? t : 0.0f;
        R[v] = rv;
        loc += rv;
      }
      const double tot = block_sum<kMdThreads>(loc, s_red);
      if (tid == 0) {
        s_Rn = tot;  // tot > 0 whenever a draft is rejected at tau (its token had R < Q~)
        s_H[s_nH++] = x[tau];
        s_qH += static_cast<double>(prob_d(tau, x[tau]));
      }
    }
    __syncthreads();
  }

  // Correction token: race over P_L (whole block accepted) or over R at tau.
  const int tau = s_tau;
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
  const int nblk = (V + 3) / 4;
  for (int gi = tid; gi < nblk; gi += kMdThreads) {
    const uint4 rnd = keyed_block(p.seed, p.step, kTagMdGumbel, b, 0, tau, gi);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int v = 4 * gi + w;
      if (v >= V) break;
      const float wt = tau == L ? prob_t(L, v) : R[v];
      if (!(wt > 0.0f)) continue;
      const float e = exponential_from_bits(word_of(rnd, w));
      if (race_better(wt, e, v, bw, be, bi)) {
        bw = wt;
        be = e;
        bi = v;
      }
    }
  }
  race_reduce<kMdThreads>(bw, be, bi, s_race);
  if (tid == 0) {
    const int a = s_a;
    for (int i = 0; i <= L; ++i) tok[i] = i < tau ? s_x[a * L + i] : (i == tau ? bi : -1);
    p.accept_len[b] = tau;
    if (p.out_draft_index) p.out_draft_index[b] = a;
  }
}

int launch_multi(const void* target, const void* draft, const int32_t* tokens,
                 const float* temps, int B, int K, int L, int V, int dtype, uint64_t seed,
                 uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                 int32_t* out_draft_index, void* workspace, const Layout& lay,
                 cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  Pass1Params p1{};
  p1.target = target;
  p1.draft = draft;
  p1.tokens = tokens;
  p1.temps = temps;
  p1.B = B;
  p1.gamma = L;
  p1.V = V;
  p1.nc = lay.nc;
  p1.rps = 2 * L + 1;
  p1.seed = seed;
  p1.step = static_cast<uint32_t>(step);
  p1.part = reinterpret_cast<RowPartial*>(ws + lay.part1);
  p1.ticket = reinterpret_cast<unsigned*>(ws + lay.ticket1);
  p1.rowstat = reinterpret_cast<RowPartial*>(ws + lay.rowstat);
  const long long grid1 = static_cast<long long>(B) * p1.rps * lay.nc;
  if (grid1 > INT_MAX)
    return set_error(SV_ERR_INVALID_ARG, "B x (2L+1) x V too large for one launch (%lld CTAs)", grid1);
  if (dtype == SV_BF16)
    pass1_multi_kernel<true><<<static_cast<unsigned>(grid1), kP1Threads, 0, stream>>>(p1);
  else
    pass1_multi_kernel<false><<<static_cast<unsigned>(grid1), kP1Threads, 0, stream>>>(p1);
  if (int rc = check_launch("multidraft pass1")) return rc;

  MdParams pm{};
  pm.target = target;
  pm.draft = draft;
  pm.tokens = tokens;
  pm.temps = temps;
  pm.B = B;
  pm.K = K;
  pm.L = L;
  pm.V = V;
  pm.seed = seed;
  pm.step = static_cast<uint32_t>(step);
  pm.rowstat = p1.rowstat;
  pm.R = reinterpret_cast<float*>(ws + lay.resid);
  pm.accept_len = out_accept_len;
  pm.out_tokens = out_tokens;
  pm.out_draft_index = out_draft_index;
  if (dtype == SV_BF16)
    md_gbv_kernel<true><<<B, kMdThreads, 0, stream>>>(pm);
  else
    md_gbv_kernel<false><<<B, kMdThreads, 0, stream>>>(pm);
  return check_launch("multidraft gbv");
}

}  // namespace sv
