// sv_single.cu -- single-draft verification: one fused, warp-specialised
// launch per call.
//
// Row statistics (FlashSpec, Methodology s.1): every target and draft row is
// streamed once; per row the maximum and the temperature-scaled softmax sum
// are reduced, and the draft token's two logits are picked up on the way.
// Decision: the CTA that completes a sequence's rows gathers the two
// log-probabilities of every draft token, draws the Philox acceptance
// uniforms and finds the first rejection with a warp ballot (FlexDraft,
// Problem definition).  Draw (Speculative Speculative Decoding, s.2 Saguaro
// sampling): the correction token comes from max(p_j - q_j, 0), the bonus
// token from p_gamma, by an exponential race with Philox noise keyed per
// vocabulary entry, split over CTAs; the last one combines.
//
// Work is handed out in queue order through a global counter: all row items
// of a sequence come before its draw items (by `lag` sequences), so whoever
// waits for a sequence's decision waits only for items that running CTAs have
// already taken and that never wait themselves; progress does not depend on
// how many CTAs are resident.  In each CTA one producer warp takes items,
// describes them and stages their logits into a ring of shared-memory stages
// with 1-D bulk copies (TMA engine); for a draw item it first waits for the
// sequence's decision.  Eight consumer warps reduce the staged rows, publish
// per-item partials, make decisions and run the draws from the staged chunks.
// Every wait is bounded in time; on expiry the kernel records an error bit in
// the workspace header and stops taking work.
#include <climits>
#include <mutex>

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"
#include "sv_stream.cuh"

namespace sv {

// Acceptance probability min(1, p/q) from log-probabilities (fp64); q = 0
// accepts when p > 0, 0/0 rejects.
__device__ __forceinline__ double accept_prob(double lp, double lq) {
  if (lq == -INFINITY) return lp == -INFINITY ? 0.0 : 1.0;
  const double r = exp(lp - lq);
  return r < 1.0 ? r : 1.0;
}

// Warp 0 of the last-arriving CTA: validate, accept/reject, write outputs.
template <bool kBf16>
__device__ __noinline__ void decide_single(const Pass1Params& p, int b, const RowAcc* rows,
                                           const float* zsel) {
  const int lane = threadIdx.x & 31;
  const int g = p.gamma;
  const float T = __ldg(p.temps + b);
  const bool tvalid = (T >= 0.0f) && !isinf(T);
  const int32_t* x = p.tokens + static_cast<size_t>(b) * g;
  int32_t* tok = p.out_tokens + static_cast<size_t>(b) * (g + 1);

  bool ok = tvalid;
  int xi[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    if (i < g) {
      xi[h] = __ldg(x + i);
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
    for (int i = lane; i <= g; i += 32) tok[i] = -1;
    for (int i = lane; i < g; i += 32) {
      if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
      if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
    }
    if (lane == 0) {
      p.accept_len[b] = -1;
      p.info[b].mode = kModeNone;
      if (p.flag) {
        __threadfence();
        store_release(p.flag + static_cast<size_t>(b) * kFlagStride, 2u);
      }
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
        const uint4 rnd = keyed_block(p.seed, p.step, kTagAccept, b, 0, i, i);
        const double u = accept_uniform(rnd.x);
        reject = !(u < accept_prob(lp, lq));
        if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = static_cast<float>(lp);
        if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = static_cast<float>(lq);
      }
      rej[h] = __ballot_sync(0xffffffffu, reject);
    }
  }
  const int j = rej[0] ? __ffs(rej[0]) - 1 : (rej[1] ? 32 + __ffs(rej[1]) - 1 : g);

  for (int i = lane; i <= g; i += 32) tok[i] = i < j ? x[i] : -1;
  if (T == 0.0f) {
    for (int i = lane; i < g; i += 32) {
      if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
      if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
    }
  }
  __syncwarp();
  if (lane == 0) {
    p.accept_len[b] = j;
    SeqInfo si{};
    if (T == 0.0f) {
      tok[j] = rows[j].arg;
      si.mode = kModeNone;
    } else {
      const float c = __fdiv_rn(kLog2e, T);
      si.mode = j < g ? kModeResidual : kModeBonus;
      si.j = j;
      si.c = c;
      si.zmp = rows[j].m;
      si.isp = __frcp_rn(rows[j].s);
      if (j < g) {
        si.zmq = rows[g + 1 + j].m;
        si.isq = __frcp_rn(rows[g + 1 + j].s);
      }
    }
    p.info[b] = si;
    if (p.flag) {
      __threadfence();
      store_release(p.flag + static_cast<size_t>(b) * kFlagStride, si.mode == kModeNone ? 2u : 1u);
    }
  }
}


// ------------------------------------------------------------------ layout
constexpr int kConsumers = kP1Threads;          // 8 consumer warps
constexpr int kFusedThreads = kConsumers + 32;  // + 1 producer warp
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = 2 * kStageVec * 16;  // target + draft piece (2 x 16 KB)
constexpr uint64_t kWaitLimitNs = 2000000000ull;      // 2 s
static_assert(kP1Threads == kP2Threads, "draw items run on the consumer warps");

// Vocabulary entries per draw item: a multiple of 4 (whole Philox blocks)
// that still fits a stage after rounding out to 16-byte vectors.
__host__ __device__ constexpr int draw_chunk(bool bf16) {
  return ((kStageVec - 2) * (bf16 ? 8 : 4)) / 4 * 4;
}

struct FusedParams {
  Pass1Params p1;             // inputs, outputs, decision state
  RacePartial* part2;         // [B][nc2] draw partials
  unsigned* ticket2;          // [B] draw arrivals
  int nc2;                    // draw items per sequence
  unsigned long long* head;   // queue position
  unsigned* exited;           // CTAs that left the queue
  unsigned* error;            // error bits
  long long n1, n2;           // row items / draw items
  int a;                      // row items per sequence ((gamma + 1) * nseg)
  int lag;                    // min(lag, B)
  int nseg;                   // vocabulary segments per row pair
  float4* pairpart;           // [B][gamma + 1][nseg] x {target, draft} partials
  float* zx;                  // [B][gamma][nseg][2] draft token's target / draft logit
};

// Queue position -> (kind, b, x): kind 1 = row item x of sequence b, kind 2 =
// draw item x of sequence b.  The queue is: row items of sequences [0, lag),
// then for k = 0..B-lag-1 the row items of sequence k+lag followed by the
// draw items of sequence k, then the draw items of the last lag sequences.
__device__ __forceinline__ void map_item(const FusedParams& f, long long q, int& kind, int& b,
                                         int& x) {
  const long long a = f.a, c2 = f.nc2, B = f.p1.B, lg = f.lag;
  if (q < lg * a) {
    kind = 1;
    b = static_cast<int>(q / a);
    x = static_cast<int>(q % a);
    return;
  }
  q -= lg * a;
  const long long unit = a + c2, nunit = B - lg;
  if (q < nunit * unit) {
    const long long k = q / unit, off = q % unit;
    if (off < a) {
      kind = 1;
      b = static_cast<int>(k + lg);
      x = static_cast<int>(off);
    } else {
      kind = 2;
      b = static_cast<int>(k);
      x = static_cast<int>(off - a);
    }
    return;
  }
  q -= nunit * unit;
  kind = 2;
  b = static_cast<int>(nunit + q / c2);
  x = static_cast<int>(q % c2);
}

template <bool kBf16>
__device__ __forceinline__ const char* target_row(const FusedParams& f, int b, int i) {
  constexpr size_t es = kBf16 ? 2 : 4;
  return static_cast<const char*>(f.p1.target) +
         (static_cast<size_t>(b) * (f.p1.gamma + 1) + i) * static_cast<size_t>(f.p1.V) * es;
}
template <bool kBf16>
__device__ __forceinline__ const char* draft_row(const FusedParams& f, int b, int i) {
  constexpr size_t es = kBf16 ? 2 : 4;
  return static_cast<const char*>(f.p1.draft) +
         (static_cast<size_t>(b) * f.p1.gamma + i) * static_cast<size_t>(f.p1.V) * es;
}

// Wait for phase `parity` of `bar`, at most kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* error) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) {
      atomicOr(error, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// What the producer tells the consumers about one stage; computed once per
// item, so the consumers do no index arithmetic of their own.
struct StageDesc {
  int kind;  // 0 = end of work, 1 = row piece, 2 = draw chunk
  int b, x;  // sequence; row item: position i; draw item: chunk
  int t, nst;
  // row pieces
  int seg, modeA, loadB, nA, nB, vA, edges, gA, gB, xg;
  float c;  // log2(e) / T
  // draw chunks
  int draw, mode2, j, e0, e1, sbA, sbB, nvA, nvB;
  float zmp, zmq, isp, isq;
};

// Producer side of a draw item: wait for the decision, then stage the
// target (and, for a residual, draft) logits of the chunk.
template <bool kBf16>
__device__ __forceinline__ void describe_draw(const FusedParams& f, int b, int chunk,
                                              StageDesc& d, const char*& rpA, const char*& rpB,
                                              int& kA, int& kB) {
  d.draw = 0;
  rpA = rpB = nullptr;
  const unsigned* flag = f.p1.flag + static_cast<size_t>(b) * kFlagStride;
  unsigned v = load_acquire(flag);
  if (v == 0) {
    const uint64_t t0 = global_ns();
    unsigned nap = 32;
    while ((v = load_acquire(flag)) == 0) {
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(f.error, kErrWaitTimeout);
        return;
      }
      __nanosleep(nap);
      if (nap < 1024) nap *= 2;
    }
  }
  if (v != 1) return;  // greedy or invalid sequence: nothing to draw
  const float4* ip = reinterpret_cast<const float4*>(f.p1.info + b);
  const float4 w0 = __ldcg(ip), w1 = __ldcg(ip + 1);
  const int mode = __float_as_int(w0.x), j = __float_as_int(w0.y);
  const int g = f.p1.gamma, V = f.p1.V;
  if (!((mode == kModeResidual && j >= 0 && j < g) || (mode == kModeBonus && j == g))) return;
  d.draw = 1;
  d.mode2 = mode;
  d.j = j;
  d.zmp = w0.z;
  d.zmq = w0.w;
  d.c = w1.x;
  d.isp = w1.y;
  d.isq = w1.z;
  constexpr int kN = Vec16<kBf16>::kN;
  d.e0 = chunk * draw_chunk(kBf16);
  d.e1 = min(V, d.e0 + draw_chunk(kBf16));
  auto span = [&](const char* rp, int& sb, int& nv, int& k0) {
    const RowGeom<kBf16> gm(rp, V);
    const int lo = max(d.e0, gm.head), hi = min(d.e1, gm.tail0);
    if (hi <= lo) {
      sb = 0;
      nv = 0;
      k0 = 0;
      return;
    }
    k0 = (lo - gm.head) / kN;
    const int k1 = (hi - gm.head + kN - 1) / kN;
    sb = gm.head + k0 * kN;
    nv = k1 - k0;
  };
  rpA = target_row<kBf16>(f, b, j);
  span(rpA, d.sbA, d.nvA, kA);
  if (mode == kModeResidual) {
    rpB = draft_row<kBf16>(f, b, j);
    span(rpB, d.sbB, d.nvB, kB);
  } else {
    d.nvB = 0;
  }
}

// The 4 logits of Philox block g (entries 4g..4g+3) of a draw row: from the
// staged chunk, or from global memory for entries outside it (a row's
// unaligned head and tail); entries at or beyond V read as -inf.
template <bool kBf16>
__device__ __forceinline__ void draw_block(const uint4* sm, int sb, int nv, const char* rp, int V,
                                           int g, float (&z)[4]) {
  constexpr int kN = Vec16<kBf16>::kN;
  const int v0 = 4 * g;
  const int off = v0 - sb;
  if (off >= 0 && off + 4 <= nv * kN && (off & 3) == 0) {
    if constexpr (kBf16) {
      const uint2 r = reinterpret_cast<const uint2*>(sm)[off >> 2];
      z[0] = bf16_lo(r.x);
      z[1] = bf16_hi(r.x);
      z[2] = bf16_lo(r.y);
      z[3] = bf16_hi(r.y);
    } else {
      const float4 r = reinterpret_cast<const float4*>(sm)[off >> 2];
      z[0] = r.x;
      z[1] = r.y;
      z[2] = r.z;
      z[3] = r.w;
    }
    return;
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int v = v0 + w, o = v - sb;
    if (v >= V) {
      z[w] = -INFINITY;
    } else if (o >= 0 && o < nv * kN) {
      if constexpr (kBf16)
        z[w] = __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(sm)[o]) << 16);
      else
        z[w] = reinterpret_cast<const float*>(sm)[o];
    } else {
      z[w] = logit_at<kBf16>(rp, v);
    }
  }
}

// Exponential race over blocks [g0, g1) (w_v / E_v, E_v = -ln U_v): w =
// max(p - q, 0) for a residual, w = 2^{(z - max) c} for a bonus.  A
// candidate is skipped without its logarithm when even the bound
// E_v >= 1 - U_v cannot beat the current best.
template <bool kBf16>
__device__ __forceinline__ void race_staged(const FusedParams& f, const StageDesc& d, int b,
                                            const uint4* smA, const uint4* smB, int g0, int g1,
                                            float& bw, float& be, int& bi) {
  const bool resid = d.mode2 == kModeResidual;
  const char* rpA = target_row<kBf16>(f, b, d.j);
  const char* rpB = resid ? draft_row<kBf16>(f, b, d.j) : rpA;
  const int V = f.p1.V;
  for (int g = g0 + static_cast<int>(threadIdx.x); g < g1; g += kConsumers) {
    float zt[4], zd[4];
    draw_block<kBf16>(smA, d.sbA, d.nvA, rpA, V, g, zt);
    if (resid) draw_block<kBf16>(smB, d.sbB, d.nvB, rpB, V, g, zd);
    const uint4 rnd = keyed_block(f.p1.seed, f.p1.step, kTagGumbel, b, 0, d.j, g);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float wt = ex2_approx((zt[w] - d.zmp) * d.c);
      if (resid) wt = wt * d.isp - ex2_approx((zd[w] - d.zmq) * d.c) * d.isq;
      if (!(wt > 0.0f)) continue;
      const uint32_t x = word_of(rnd, w);
      if (bw > 0.0f && wt * be <= bw * gumbel_one_minus_u(x)) continue;
      const float e = exponential_from_bits(x);
      const int v = 4 * g + w;
      if (race_better(wt, e, v, bw, be, bi)) {
        bw = wt;
        be = e;
        bi = v;
      }
    }
  }
}

// Fallback draw over a whole target row from global memory (the residual
// vanished: p_j == q_j to rounding), run by the consumers of one CTA.
template <bool kBf16>
__device__ void race_row_global(const FusedParams& f, const StageDesc& d, int b, float& bw,
                                float& be, int& bi) {
  const char* rp = target_row<kBf16>(f, b, d.j);
  const int V = f.p1.V;
  for (int g = threadIdx.x; g < (V + 3) / 4; g += kConsumers) {
    const uint4 rnd = keyed_block(f.p1.seed, f.p1.step, kTagGumbel, b, 0, d.j, g);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int v = 4 * g + w;
      if (v >= V) break;
      const float wt = ex2_approx((logit_at<kBf16>(rp, v) - d.zmp) * d.c);
      if (!(wt > 0.0f)) continue;
      const float e = exponential_from_bits(word_of(rnd, w));
      if (race_better(wt, e, v, bw, be, bi)) {
        bw = wt;
        be = e;
        bi = v;
      }
    }
  }
}

// Reduce the two rows' accumulators over the consumer threads (one barrier);
// the result is valid in thread 0.
__device__ __forceinline__ void reduce_pair(RowAcc& A, RowAcc& B, int modeA, float c,
                                            RowAcc* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    RowAcc oa, ob;
    oa.m = __shfl_down_sync(0xffffffffu, A.m, off);
    oa.s = __shfl_down_sync(0xffffffffu, A.s, off);
    oa.arg = __shfl_down_sync(0xffffffffu, A.arg, off);
    oa.bad = __shfl_down_sync(0xffffffffu, A.bad, off);
    ob.m = __shfl_down_sync(0xffffffffu, B.m, off);
    ob.s = __shfl_down_sync(0xffffffffu, B.s, off);
    ob.bad = __shfl_down_sync(0xffffffffu, B.bad, off);
    ob.arg = 0x7fffffff;
    if (modeA == kRowArgmax) acc_merge<kRowArgmax>(A, oa, c); else acc_merge<kRowLse>(A, oa, c);
    acc_merge<kRowLse>(B, ob, c);
  }
  if (lane == 0) {
    scratch[2 * warp] = A;
    scratch[2 * warp + 1] = B;
  }
  block_sync<kConsumers>();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kConsumers / 32; ++w) {
      if (modeA == kRowArgmax) acc_merge<kRowArgmax>(A, scratch[2 * w], c);
      else acc_merge<kRowLse>(A, scratch[2 * w], c);
      acc_merge<kRowLse>(B, scratch[2 * w + 1], c);
    }
  }
}

// Combine the nseg pair partials of every position of sequence b into the
// row table rows[] (target rows 0..gamma, then draft rows), and pick up the
// draft tokens' logits (zsel[2i], zsel[2i+1]).
__device__ __forceinline__ void combine_pairs(const FusedParams& f, int b, RowAcc* rows,
                                              float* zsel) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = f.p1.gamma;
  const float T = __ldg(f.p1.temps + b);
  const int modeA = row_mode(T, true);
  const float c = modeA == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
  for (int i = warp; i <= g; i += kConsumers / 32) {
    RowAcc A{-INFINITY, 0.0f, 0x7fffffff, 0}, B{-INFINITY, 0.0f, 0x7fffffff, 0};
    const float4* pp = f.pairpart + (static_cast<size_t>(b) * (g + 1) + i) * f.nseg * 2;
    for (int q = lane; q < f.nseg; q += 32) {
      const float4 a = __ldcg(pp + 2 * q), d = __ldcg(pp + 2 * q + 1);
      const RowAcc oa{a.x, a.y, __float_as_int(a.z), __float_as_int(a.w)};
      const RowAcc ob{d.x, d.y, __float_as_int(d.z), __float_as_int(d.w)};
      if (modeA == kRowArgmax) acc_merge<kRowArgmax>(A, oa, c); else acc_merge<kRowLse>(A, oa, c);
      acc_merge<kRowLse>(B, ob, c);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      RowAcc oa, ob;
      oa.m = __shfl_down_sync(0xffffffffu, A.m, off);
      oa.s = __shfl_down_sync(0xffffffffu, A.s, off);
      oa.arg = __shfl_down_sync(0xffffffffu, A.arg, off);
      oa.bad = __shfl_down_sync(0xffffffffu, A.bad, off);
      ob.m = __shfl_down_sync(0xffffffffu, B.m, off);
      ob.s = __shfl_down_sync(0xffffffffu, B.s, off);
      ob.bad = __shfl_down_sync(0xffffffffu, B.bad, off);
      ob.arg = 0x7fffffff;
      if (modeA == kRowArgmax) acc_merge<kRowArgmax>(A, oa, c); else acc_merge<kRowLse>(A, oa, c);
      acc_merge<kRowLse>(B, ob, c);
    }
    if (lane == 0) {
      rows[i] = A;
      if (i < g) rows[g + 1 + i] = B;
    }
    if (i < g) {
      // the draft token's logits: the one segment that holds it reports them
      float zt = __int_as_float(0x7fc00000), zd = zt;
      const float* zp = f.zx + (static_cast<size_t>(b) * g + i) * f.nseg * 2;
      for (int q = lane; q < f.nseg; q += 32) {
        const float a = __ldcg(zp + 2 * q), d = __ldcg(zp + 2 * q + 1);
        if (a == a) zt = a;
        if (d == d) zd = d;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float a = __shfl_down_sync(0xffffffffu, zt, off);
        const float d = __shfl_down_sync(0xffffffffu, zd, off);
        if (zt != zt) zt = a;
        if (zd != zd) zd = d;
      }
      if (lane == 0) {
        zsel[2 * i] = zt;
        zsel[2 * i + 1] = zd;
      }
    }
  }
  block_sync<kConsumers>();
}

template <bool kBf16>
__device__ __forceinline__ void row_edges(const FusedParams& f, const char* rp, int mode, float c,
                                          bool head, bool tail, int xg, float* zx, RunAcc& acc) {
  const RowGeom<kBf16> g(rp, f.p1.V);
  const int tid = threadIdx.x;
  if (head)
    for (int v = tid; v < g.head; v += kConsumers) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) *zx = z;
      if (mode == kRowLse) lse_scalar(acc, z, c); else argmax_scalar(acc, z, v);
    }
  if (tail)
    for (int v = g.tail0 + tid; v < f.p1.V; v += kConsumers) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) *zx = z;
      if (mode == kRowLse) lse_scalar(acc, z, c); else argmax_scalar(acc, z, v);
    }
}

// ----------------------------------------------------------------- kernel
template <bool kBf16>
__global__ void __launch_bounds__(kFusedThreads, 2) fused_single_kernel(FusedParams f) {
  extern __shared__ __align__(128) uint4 stage[];  // kStages x (2 x kStageVec) vectors
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ StageDesc desc[kStages];
  __shared__ RowAcc rows[kMaxRowsPerSeq];
  __shared__ RowAcc scratch[2 * (kConsumers / 32)];
  __shared__ float4 race_scratch[kConsumers / 32];
  __shared__ int s_last;
  __shared__ float s_zx[2];                   // the draft token's logits in the current row item
  __shared__ float s_zsel[2 * SV_MAX_GAMMA];  // per position, for the decision
  __shared__ volatile int s_abort;
  // Wait for the previous grid in the stream (programmatic dependent launch),
  // then let the next one start launching its CTAs.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const long long total = f.n1 + f.n2;
  const int tid = threadIdx.x;
  constexpr int kN = Vec16<kBf16>::kN;
  constexpr size_t kStride = 2 * kStageVec;  // vectors per stage
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);  // one arrival per consumer warp
    }
    mbar_fence_init();
    s_abort = 0;
    s_zx[0] = s_zx[1] = __int_as_float(0x7fc00000);
  }
  __syncthreads();

  if (tid >= kConsumers) {
    // ---------------- producer warp (one lane) ----------------
    if (tid != kConsumers) return;
    uint32_t emask = (1u << kStages) - 1;  // a fresh barrier's "previous" phase is complete
    int s = 0;
    long long q = static_cast<long long>(atomicAdd(f.head, 1ull));
    for (;;) {
      // take the next position now; its latency overlaps this item's staging
      const long long qn = q < total ? static_cast<long long>(atomicAdd(f.head, 1ull)) : total;
      StageDesc d{};
      const char *rpA = nullptr, *rpB = nullptr;
      int a0 = 0, a1 = 0, b0 = 0, b1 = 0, headA = 0, headB = 0, kA = 0, kB = 0;
      d.nst = 1;
      if (q < total) {
        int kind, b, x;
        map_item(f, q, kind, b, x);
        d.kind = kind;
        d.b = b;
        d.x = x;
        if (kind == 1) {
          const float T = __ldg(f.p1.temps + b);
          const int i = x / f.nseg;
          d.x = i;
          d.seg = x - i * f.nseg;
          d.modeA = row_mode(T, true);
          d.loadB = i < f.p1.gamma && row_mode(T, false) == kRowLse;
          d.c = d.modeA == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
          d.xg = -1;
          if (d.modeA == kRowLse && i < f.p1.gamma) {
            const int xt = __ldg(f.p1.tokens + static_cast<size_t>(b) * f.p1.gamma + i);
            if (xt >= 0 && xt < f.p1.V) d.xg = xt;
          }
          int n = 0;
          if (d.modeA != kRowSkip) {
            rpA = target_row<kBf16>(f, b, i);
            const RowGeom<kBf16> g(rpA, f.p1.V);
            g.segment(d.seg, f.nseg, a0, a1);
            headA = g.head;
            n = (a1 - a0 + kStageVec - 1) / kStageVec;
          }
          if (d.loadB) {
            rpB = draft_row<kBf16>(f, b, i);
            const RowGeom<kBf16> g(rpB, f.p1.V);
            g.segment(d.seg, f.nseg, b0, b1);
            headB = g.head;
            n = max(n, (b1 - b0 + kStageVec - 1) / kStageVec);
          }
          d.nst = n < 1 ? 1 : n;
        } else {
          describe_draw<kBf16>(f, b, x, d, rpA, rpB, kA, kB);
        }
      }
      for (int t = 0; t < d.nst; ++t) {
        if (s_abort || !mbar_wait(&empty[s], (emask >> s) & 1u, f.error)) {
          s_abort = 1;  // the consumers stop at their next stage
          return;
        }
        emask ^= 1u << s;
        StageDesc e = d;
        e.t = t;
        uint4* st = stage + s * kStride;
        uint32_t bytesA = 0, bytesB = 0;
        const void *srcA = nullptr, *srcB = nullptr;
        if (d.kind == 1) {
          const int ka = min(a1, a0 + t * kStageVec), kb = min(b1, b0 + t * kStageVec);
          e.nA = rpA ? min(a1, ka + kStageVec) - ka : 0;
          e.nB = rpB ? min(b1, kb + kStageVec) - kb : 0;
          const int baseA = headA + ka * kN, baseB = headB + kb * kN;
          e.vA = baseA;
          e.gA = (d.xg >= baseA && d.xg < baseA + e.nA * kN) ? d.xg - baseA : -1;
          e.gB = (d.xg >= baseB && d.xg < baseB + e.nB * kN) ? d.xg - baseB : -1;
          const bool first = d.seg == 0 && t == 0, last = d.seg == f.nseg - 1 && t == d.nst - 1;
          e.edges = (rpA && first ? 1 : 0) | (rpA && last ? 2 : 0) | (rpB && first ? 4 : 0) |
                    (rpB && last ? 8 : 0);
          bytesA = static_cast<uint32_t>(e.nA) * 16u;
          bytesB = static_cast<uint32_t>(e.nB) * 16u;
          if (bytesA) srcA = rpA + static_cast<size_t>(headA) * (kBf16 ? 2 : 4) + static_cast<size_t>(ka) * 16;
          if (bytesB) srcB = rpB + static_cast<size_t>(headB) * (kBf16 ? 2 : 4) + static_cast<size_t>(kb) * 16;
        } else if (d.kind == 2 && d.draw) {
          bytesA = static_cast<uint32_t>(d.nvA) * 16u;
          bytesB = static_cast<uint32_t>(d.nvB) * 16u;
          if (bytesA) srcA = rpA + static_cast<size_t>(d.sbA) * (kBf16 ? 2 : 4);
          if (bytesB) srcB = rpB + static_cast<size_t>(d.sbB) * (kBf16 ? 2 : 4);
        }
        desc[s] = e;
        if (bytesA + bytesB) {
          fence_proxy_async_smem();  // the stage was last read through the generic proxy
          mbar_expect_tx(&full[s], bytesA + bytesB);
          if (bytesA) bulk_load(st, srcA, bytesA, &full[s]);
          if (bytesB) bulk_load(st + kStageVec, srcB, bytesB, &full[s]);
        } else {
          mbar_arrive(&full[s]);
        }
        s = (s + 1) % kStages;
      }
      if (q >= total) return;  // the end-of-work stage has been published
      q = qn;
    }
  }

  // ---------------- consumer warps ----------------
  uint32_t fmask = 0u;
  int s = 0;
  // Thread 0 waits (bounded); the barrier makes the abort decision uniform;
  // then every consumer acquires the stage.
  auto wait_stage = [&]() -> bool {
    if (tid == 0 && !mbar_wait(&full[s], (fmask >> s) & 1u, f.error)) s_abort = 1;
    block_sync<kConsumers>();
    if (s_abort) return false;
    mbar_try_wait(&full[s], (fmask >> s) & 1u);
    fmask ^= 1u << s;
    return true;
  };
  auto release_stage = [&]() {
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&empty[s]);
    s = (s + 1) % kStages;
  };
  for (;;) {
    if (!wait_stage()) break;
    const int kind = desc[s].kind;
    if (kind == 0) break;
    const int b = desc[s].b, x = desc[s].x;
    if (kind == 1) {
      // ---- row item: target row x and draft row x over one segment ----
      const int seg = desc[s].seg, nst = desc[s].nst, modeA = desc[s].modeA;
      const float c = desc[s].c;
      RunAcc accA, accB;
      accA.reset();
      accB.reset();
      for (int t = 0;;) {
        const StageDesc& d = desc[s];
        const uint4* sm = stage + s * kStride;
        constexpr int kR = kStageVec / kConsumers;  // vectors per thread per row piece
        {
          uint4 ra[kR];
          const int na = d.nA > tid ? (d.nA - tid + kConsumers - 1) / kConsumers : 0;
#pragma unroll
          for (int j = 0; j < kR; ++j)
            if (j < na) ra[j] = sm[tid + j * kConsumers];
#pragma unroll
          for (int j = 0; j < kR; ++j)  // compile-time j keeps ra[] in registers
            if (d.gA >= 0 && d.gA / kN == tid + j * kConsumers) s_zx[0] = Vec16<kBf16>::at(ra[j], d.gA % kN);
          if (modeA == kRowLse) {
            lse_block<kBf16, kR>(accA, ra, na, c);
          } else if (modeA == kRowArgmax) {
            int v0[kR];
#pragma unroll
            for (int j = 0; j < kR; ++j) v0[j] = d.vA + (tid + j * kConsumers) * kN;
            argmax_block<kBf16, kR>(accA, ra, na, v0);
          }
        }
        {
          uint4 rb[kR];
          const int nb = d.nB > tid ? (d.nB - tid + kConsumers - 1) / kConsumers : 0;
#pragma unroll
          for (int j = 0; j < kR; ++j)
            if (j < nb) rb[j] = sm[kStageVec + tid + j * kConsumers];
#pragma unroll
          for (int j = 0; j < kR; ++j)
            if (d.gB >= 0 && d.gB / kN == tid + j * kConsumers) s_zx[1] = Vec16<kBf16>::at(rb[j], d.gB % kN);
          lse_block<kBf16, kR>(accB, rb, nb, c);
        }
        const int edges = d.edges, xg = d.xg;
        release_stage();  // desc[] of this stage is not read past this point
        if (edges & 3)
          row_edges<kBf16>(f, target_row<kBf16>(f, b, x), modeA, c, edges & 1, edges & 2, xg, &s_zx[0], accA);
        if (edges & 12)
          row_edges<kBf16>(f, draft_row<kBf16>(f, b, x), kRowLse, c, edges & 4, edges & 8, xg, &s_zx[1], accB);
        if (++t == nst) break;
        if (!wait_stage()) break;
      }
      if (s_abort) break;
      // ---- finalize: reduce, publish, take the sequence's ticket ----
      RowAcc A = accA.row(), B = accB.row();
      reduce_pair(A, B, modeA, c, scratch);
      if (tid == 0) {
        float4* pp = f.pairpart + ((static_cast<size_t>(b) * (f.p1.gamma + 1) + x) * f.nseg + seg) * 2;
        pp[0] = make_float4(A.m, A.s, __int_as_float(A.arg), __int_as_float(A.bad));
        pp[1] = make_float4(B.m, B.s, __int_as_float(B.arg), __int_as_float(B.bad));
        if (x < f.p1.gamma) {
          float* z = f.zx + ((static_cast<size_t>(b) * f.p1.gamma + x) * f.nseg + seg) * 2;
          z[0] = s_zx[0];
          z[1] = s_zx[1];
        }
        s_zx[0] = s_zx[1] = __int_as_float(0x7fc00000);  // NaN: "not in this segment"
        const unsigned tk = ticket_release(f.p1.ticket + b);
        s_last = (tk == static_cast<unsigned>(f.a - 1));
        if (s_last) f.p1.ticket[b] = 0;  // leave the counter at zero for the next call
      }
      block_sync<kConsumers>();
      if (s_last) {
        fence_acquire();
        combine_pairs(f, b, rows, s_zsel);
        if (tid < 32) decide_single<kBf16>(f.p1, b, rows, s_zsel);
        block_sync<kConsumers>();  // rows[] / s_last are reused by the next item
      }
    } else {
      // ---- draw item: race over the staged chunk ----
      const StageDesc d = desc[s];  // copy: the stage is released before the combine
      float bw = 0.0f, be = 1.0f;
      int bi = INT_MAX;
      if (d.draw) {
        const uint4* sm = stage + s * kStride;
        race_staged<kBf16>(f, d, b, sm, sm + kStageVec, d.e0 / 4, (d.e1 + 3) / 4, bw, be, bi);
      }
      release_stage();
      race_reduce<kConsumers>(bw, be, bi, race_scratch);
      if (tid == 0) {
        RacePartial* pp = f.part2 + static_cast<size_t>(b) * f.nc2 + x;
        *reinterpret_cast<float4*>(pp) = make_float4(bw, be, __int_as_float(bi), 0.0f);
        const unsigned tk = ticket_release(f.ticket2 + b);
        s_last = (tk == static_cast<unsigned>(f.nc2 - 1));
        if (s_last) f.ticket2[b] = 0;
      }
      block_sync<kConsumers>();
      if (s_last) {
        fence_acquire();
        if (d.draw) {
          bw = 0.0f;
          be = 1.0f;
          bi = INT_MAX;
          for (int q = tid; q < f.nc2; q += kConsumers) {
            const float4 g = __ldcg(reinterpret_cast<const float4*>(f.part2 + static_cast<size_t>(b) * f.nc2 + q));
            if (race_better(g.x, g.y, __float_as_int(g.z), bw, be, bi)) {
              bw = g.x;
              be = g.y;
              bi = __float_as_int(g.z);
            }
          }
          race_reduce<kConsumers>(bw, be, bi, race_scratch);
          if (!(bw > 0.0f)) {  // uniform: race_reduce returns the winner to every thread
            bw = 0.0f;
            be = 1.0f;
            bi = INT_MAX;
            race_row_global<kBf16>(f, d, b, bw, be, bi);
            race_reduce<kConsumers>(bw, be, bi, race_scratch);
          }
          if (tid == 0) f.p1.out_tokens[static_cast<size_t>(b) * (f.p1.gamma + 1) + d.j] = bi;
        }
        if (tid == 0) f.p1.flag[static_cast<size_t>(b) * kFlagStride] = 0u;  // all readers are done
        block_sync<kConsumers>();  // s_last is reused by the next item
      }
    }
  }
  block_sync<kConsumers>();
  if (tid == 0) {
    const unsigned n = atomicAdd(f.exited, 1u);
    if (n == gridDim.x - 1) {  // last CTA out leaves the queue reset
      *f.head = 0ull;
      *f.exited = 0u;
    }
  }
}

// ------------------------------------------------------------------ launch
namespace {
struct Occupancy {
  int sms = 0, per_sm[2] = {0, 0};
};
Occupancy g_occ[64];
std::mutex g_occ_mu;

int resident_ctas(bool bf16) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lk(g_occ_mu);
  Occupancy& o = g_occ[dev];
  if (o.sms == 0) cudaDeviceGetAttribute(&o.sms, cudaDevAttrMultiProcessorCount, dev);
  int& n = o.per_sm[bf16 ? 1 : 0];
  if (n == 0) {
    const int dyn = kStages * static_cast<int>(kStageBytes);
    if (bf16) {
      cudaFuncSetAttribute(fused_single_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_single_kernel<true>, kFusedThreads, dyn);
    } else {
      cudaFuncSetAttribute(fused_single_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_single_kernel<false>, kFusedThreads, dyn);
    }
    if (n < 1) n = 1;
  }
  return o.sms * n;
}
}  // namespace

int draw_chunks(int V, int dtype) {
  const int per = draw_chunk(dtype == SV_BF16);
  return (V + per - 1) / per;
}

int launch_single(const void* target, const void* draft, const int32_t* tokens,
                  const float* temps, int B, int gamma, int V, int dtype, uint64_t seed,
                  uint64_t step, int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                  float* out_lq, void* workspace, const Layout& lay, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  FusedParams f{};
  Pass1Params& p1 = f.p1;
  p1.target = target;
  p1.draft = draft;
  p1.tokens = tokens;
  p1.temps = temps;
  p1.B = B;
  p1.gamma = gamma;
  p1.V = V;
  p1.rps = 2 * gamma + 1;
  p1.seed = seed;
  p1.step = static_cast<uint32_t>(step);
  p1.ticket = reinterpret_cast<unsigned*>(ws + lay.ticket1);
  p1.info = reinterpret_cast<SeqInfo*>(ws + lay.info);
  p1.flag = reinterpret_cast<unsigned*>(ws + lay.flag);
  p1.accept_len = out_accept_len;
  p1.out_tokens = out_tokens;
  p1.out_lp = out_lp;
  p1.out_lq = out_lq;
  f.part2 = reinterpret_cast<RacePartial*>(ws + lay.part2);
  f.ticket2 = reinterpret_cast<unsigned*>(ws + lay.ticket2);
  f.nc2 = lay.nc2;
  f.head = reinterpret_cast<unsigned long long*>(ws + lay.ctl);
  f.exited = reinterpret_cast<unsigned*>(ws + lay.ctl + 8);
  f.error = reinterpret_cast<unsigned*>(ws + lay.ctl + 12);
  const bool bf16 = dtype == SV_BF16;
  const int S = resident_ctas(bf16);
  // Segments per row pair: about 8 row items per resident CTA (load
  // balance), bounded by the workspace's segment capacity.
  const long long pairs = static_cast<long long>(B) * (gamma + 1);
  long long nseg = (8LL * S + pairs - 1) / pairs;
  if (nseg > lay.nc) nseg = lay.nc;
  if (nseg < 1) nseg = 1;
  f.nseg = static_cast<int>(nseg);
  f.pairpart = reinterpret_cast<float4*>(ws + lay.part1);
  f.zx = reinterpret_cast<float*>(ws + lay.resid);
  f.a = (gamma + 1) * f.nseg;
  f.n1 = static_cast<long long>(B) * f.a;
  f.n2 = static_cast<long long>(B) * f.nc2;
  const long long items = f.n1 + f.n2;
  const unsigned grid = static_cast<unsigned>(items < S ? items : S);
  // A sequence's draw items are queued about one resident wave of items
  // after its row items: late enough that its decision is usually made, early
  // enough that its rows are usually still in L2.
  const long long lag = static_cast<long long>(grid) / f.a + 1;
  f.lag = static_cast<int>(lag < B ? lag : B);

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = kStages * kStageBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = bf16 ? cudaLaunchKernelEx(&cfg, fused_single_kernel<true>, f)
                       : cudaLaunchKernelEx(&cfg, fused_single_kernel<false>, f);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;  // retry as an ordinary stream-ordered launch
    e = bf16 ? cudaLaunchKernelEx(&cfg, fused_single_kernel<true>, f)
             : cudaLaunchKernelEx(&cfg, fused_single_kernel<false>, f);
  }
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "fused verify launch failed: %s", cudaGetErrorString(e));
  return check_launch("fused verify");
}

}  // namespace sv
