// sv_single.cu -- single-draft verification: pass 1 + decision, pass 2.
//
// Pass 1 (FlashSpec, Methodology s.1): every logit row of the step is
// streamed once; per row the temperature-scaled softmax normaliser and the
// maximum are reduced.  The CTA that finishes a sequence's last chunk makes
// that sequence's decision: it gathers the two log-probabilities of every
// draft token, draws the Philox acceptance uniforms, and finds the first
// rejection with a warp ballot (FlexDraft, Problem definition).
// Pass 2 (Speculative Speculative Decoding, s.2 Saguaro sampling): the
// correction token is drawn from max(p_j - q_j, 0), or the bonus token from
// p_gamma, by an exponential race with Philox noise keyed per vocabulary
// entry; CTAs split the vocabulary and the last one combines.
#include <climits>
#include <mutex>

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

// Warp 0 of the last-arriving CTA: validate, accept/reject, write outputs.
template <bool kBf16>
__device__ __noinline__ void decide_single(const Pass1Params& p, int b, const RowAcc* rows) {
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
        const float dp = __fsub_rn(__fdiv_rn(logit_at<kBf16>(tr, xi[h]), T), __fdiv_rn(ap.m, T));
        const float dq = __fsub_rn(__fdiv_rn(logit_at<kBf16>(dr, xi[h]), T), __fdiv_rn(aq.m, T));
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

// ---------------------------------------------------------------- pass 2
// The 4 logits of Philox block g (entries 4g..4g+3) of one row, kept packed
// until used: one 8-byte (bf16) or 16-byte (fp32) load when the row base
// allows it, otherwise scalar loads; entries at or beyond V read as -inf.
template <bool kBf16>
struct Block4;

template <>
struct Block4<true> {
  uint2 r;
  __device__ __forceinline__ void load(const char* row, bool vec_ok, int V, int g) {
    const int v0 = 4 * g;
    if (vec_ok && v0 + 3 < V) {
      r = __ldg(reinterpret_cast<const uint2*>(row) + g);
    } else {
      const uint16_t* q = reinterpret_cast<const uint16_t*>(row);
      const uint32_t ninf = 0xFF80u;  // bf16 -inf
      uint32_t h[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) h[w] = v0 + w < V ? static_cast<uint32_t>(__ldg(q + v0 + w)) : ninf;
      r = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    }
  }
  __device__ __forceinline__ float at(int w) const {
    const uint32_t x = w < 2 ? r.x : r.y;
    return (w & 1) ? bf16_hi(x) : bf16_lo(x);
  }
};

template <>
struct Block4<false> {
  float4 r;
  __device__ __forceinline__ void load(const char* row, bool vec_ok, int V, int g) {
    const int v0 = 4 * g;
    if (vec_ok && v0 + 3 < V) {
      r = __ldg(reinterpret_cast<const float4*>(row) + g);
    } else {
      const float* q = reinterpret_cast<const float*>(row);
      r.x = v0 + 0 < V ? __ldg(q + v0 + 0) : -INFINITY;
      r.y = v0 + 1 < V ? __ldg(q + v0 + 1) : -INFINITY;
      r.z = v0 + 2 < V ? __ldg(q + v0 + 2) : -INFINITY;
      r.w = v0 + 3 < V ? __ldg(q + v0 + 3) : -INFINITY;
    }
  }
  __device__ __forceinline__ float at(int w) const {
    return w == 0 ? r.x : (w == 1 ? r.y : (w == 2 ? r.z : r.w));
  }
};

// Exponential race over Philox blocks [g0, g1) of the draw row(s): the winner
// of w_v / E_v (E_v = -ln U_v) with w = max(p - q, 0) (residual) or
// w = 2^{(z - max) c} (bonus, unnormalised).  Each thread loads kU blocks
// before using any of them.  A candidate is skipped without its logarithm
// when even the bound E_v >= 1 - U_v cannot beat the current best.
template <bool kBf16>
__device__ __forceinline__ void race_block(const Pass2Params& p, const SeqInfo& si, int b, int g0,
                                           int g1, float& bw, float& be, int& bi) {
  constexpr int kU = 2;
  constexpr size_t es = kBf16 ? 2 : 4;
  constexpr uintptr_t kVecAlign = kBf16 ? 8 : 16;
  const int gmm = p.gamma;
  const char* trow = static_cast<const char*>(p.target) +
                     (static_cast<size_t>(b) * (gmm + 1) + si.j) * static_cast<size_t>(p.V) * es;
  const char* drow = static_cast<const char*>(p.draft) +
                     (static_cast<size_t>(b) * gmm + si.j) * static_cast<size_t>(p.V) * es;
  const bool resid = si.mode == kModeResidual;
  const bool tvec = (reinterpret_cast<uintptr_t>(trow) % kVecAlign) == 0;
  const bool dvec = (reinterpret_cast<uintptr_t>(drow) % kVecAlign) == 0;
  for (int gb = g0 + static_cast<int>(threadIdx.x); gb < g1; gb += kU * kP2Threads) {
    Block4<kBf16> zt[kU], zd[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int g = gb + u * kP2Threads;
      if (g < g1) {
        zt[u].load(trow, tvec, p.V, g);
        if (resid) zd[u].load(drow, dvec, p.V, g);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int g = gb + u * kP2Threads;
      if (g >= g1) break;
      const uint4 rnd = keyed_block(p.seed, p.step, kTagGumbel, b, 0, si.j, g);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        float wt = ex2_approx((zt[u].at(w) - si.zmp) * si.c);
        if (resid) wt = wt * si.isp - ex2_approx((zd[u].at(w) - si.zmq) * si.c) * si.isq;
        if (!(wt > 0.0f)) continue;
        const uint32_t x = word_of(rnd, w);
        // bound: E >= t = 1 - U, so w / E <= w / t
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
}

// ------------------------------------------------------- fused single pass
// One launch per call, warp-specialised.  Work items are handed out in queue
// order through a global counter: all pass-1 chunks of a sequence come before
// its pass-2 chunks (by `lag` sequences), so a CTA that waits for a
// sequence's decision waits only for items that running CTAs have already
// taken and that never wait themselves; progress does not depend on how many
// CTAs are resident.
//
// In each CTA one producer warp takes items from the queue and, for pass-1
// chunks, starts a 1-D bulk copy (TMA engine) of the chunk into a ring of
// kStages shared-memory stages (full/empty mbarriers); eight consumer warps
// reduce the staged chunk, publish it, make a sequence's decision when they
// complete it, and run the pass-2 draws.  The producer runs up to kStages items
// ahead, so the copies of later chunks overlap the consumers' work and their
// waits.  Every wait is bounded in time; on expiry the kernel records an
// error bit in the workspace header and stops taking work.
constexpr int kConsumers = kP1Threads;         // 8 consumer warps
constexpr int kFusedThreads = kConsumers + 32;  // + 1 producer warp
constexpr int kStages = 4;
constexpr uint32_t kStageBytes = 16384;  // one pass-1 chunk body (1024 x 16 B)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
static_assert(kP1Threads == kP2Threads, "pass-2 items run on the consumer warps");

struct FusedParams {
  Pass1Params p1;
  Pass2Params p2;
  unsigned long long* head;  // queue position
  unsigned* exited;          // CTAs that left the queue
  unsigned* error;           // error bits
  long long n1, n2;          // pass-1 / pass-2 items
  int a;                     // pass-1 items per sequence
  int lag;                   // min(lag, B)
};

// Queue position -> (kind, b, x): kind 1 = pass-1 item x of sequence b,
// kind 2 = pass-2 chunk x of sequence b.  The queue is: pass-1 items of
// sequences [0, lag), then for k = 0..B-lag-1 the pass-1 items of sequence
// k+lag followed by the pass-2 items of sequence k, then the pass-2 items of
// the last lag sequences.
__device__ __forceinline__ void map_item(const FusedParams& f, long long q, int& kind, int& b,
                                         int& x) {
  const long long a = f.a, c2 = f.p2.nc2, B = f.p1.B, lg = f.lag;
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

template <bool kBf16>
__device__ void pass2_item(const FusedParams& f, int b, int chunk, float4* scratch,
                          unsigned* s_flag, int* s_last) {
  __shared__ SeqInfo s_si;
  const Pass2Params& p = f.p2;
  unsigned* flag = f.p1.flag + static_cast<size_t>(b) * kFlagStride;
  if (threadIdx.x == 0) {
    unsigned v = load_acquire(flag);
    if (v == 0) {
      const uint64_t t0 = global_ns();
      unsigned nap = 32;
      while ((v = load_acquire(flag)) == 0) {
        if (global_ns() - t0 > kWaitLimitNs) {
          atomicOr(f.error, kErrWaitTimeout);
          v = 3;
          break;
        }
        __nanosleep(nap);
        if (nap < 1024) nap *= 2;
      }
    }
    SeqInfo si{};
    if (v == 1) {
      const float4* ip = reinterpret_cast<const float4*>(f.p1.info + b);
      const float4 w0 = __ldcg(ip), w1 = __ldcg(ip + 1);
      si.mode = __float_as_int(w0.x);
      si.j = __float_as_int(w0.y);
      si.zmp = w0.z;
      si.zmq = w0.w;
      si.c = w1.x;
      si.isp = w1.y;
      si.isq = w1.z;
      const bool ok = (si.mode == kModeResidual || si.mode == kModeBonus) && si.j >= 0 &&
                      si.j <= p.gamma && !(si.mode == kModeResidual && si.j == p.gamma);
      if (!ok) v = 3;
    }
    s_si = si;
    *s_flag = v;
  }
  block_sync<kConsumers>();
  // v and si come from shared memory: every consumer takes the same branches.
  const unsigned v = *s_flag;
  SeqInfo si = s_si;
  const bool draw = (v == 1);
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
  const int nblocks = (p.V + 3) / 4;
  if (draw) {
    const int g0 = chunk * p.blocks_per_chunk;
    const int g1 = min(nblocks, g0 + p.blocks_per_chunk);
    race_block<kBf16>(p, si, b, g0, g1, bw, be, bi);
  }
  race_reduce<kConsumers>(bw, be, bi, scratch);
  if (threadIdx.x == 0) {
    RacePartial* pp = p.part + static_cast<size_t>(b) * p.nc2 + chunk;
    *reinterpret_cast<float4*>(pp) = make_float4(bw, be, __int_as_float(bi), 0.0f);
    __threadfence();
    const unsigned t = atomicAdd(p.ticket + b, 1u);
    *s_last = (t == static_cast<unsigned>(p.nc2 - 1));
    if (*s_last) p.ticket[b] = 0;
  }
  block_sync<kConsumers>();
  if (!*s_last) return;
  __threadfence();
  if (draw) {
    bw = 0.0f;
    be = 1.0f;
    bi = INT_MAX;
    for (int q = threadIdx.x; q < p.nc2; q += kConsumers) {
      const float4 g = __ldcg(reinterpret_cast<const float4*>(p.part + static_cast<size_t>(b) * p.nc2 + q));
      if (race_better(g.x, g.y, __float_as_int(g.z), bw, be, bi)) {
        bw = g.x;
        be = g.y;
        bi = __float_as_int(g.z);
      }
    }
    race_reduce<kConsumers>(bw, be, bi, scratch);
    if (!(bw > 0.0f)) {
      si.mode = kModeBonus;  // residual vanished: draw from p_j
      bw = 0.0f;
      be = 1.0f;
      bi = INT_MAX;
      race_block<kBf16>(p, si, b, 0, nblocks, bw, be, bi);
      race_reduce<kConsumers>(bw, be, bi, scratch);
    }
    if (threadIdx.x == 0) p.out_tokens[static_cast<size_t>(b) * (p.gamma + 1) + si.j] = bi;
  }
  if (threadIdx.x == 0) *flag = 0u;  // every pass-2 CTA of b has read it
}

struct StagePlan {
  bool load;  // a pass-1 chunk whose row must be read
  int b, r, chunk, mode;
};

template <bool kBf16>
__device__ __forceinline__ StagePlan plan_item(const FusedParams& f, long long q) {
  StagePlan s{false, 0, -1, 0, kRowSkip};
  int kind, b, x;
  map_item(f, q, kind, b, x);
  s.b = b;
  if (kind != 1) {
    s.chunk = x;
    return s;
  }
  s.r = x / f.p1.nc;
  s.chunk = x - s.r * f.p1.nc;
  s.mode = row_mode(__ldg(f.p1.temps + b), s.r <= f.p1.gamma);
  s.load = s.mode != kRowSkip;
  return s;
}

// Producer: publish item q in a stage and start its copy (or just arrive).
template <bool kBf16>
__device__ __forceinline__ void produce(const FusedParams& f, long long q, long long total,
                                        uint4* stage, uint64_t* full) {
  if (q < total) {
    const StagePlan s = plan_item<kBf16>(f, q);
    if (s.load) {
      bool is_target;
      const char* rp = row_ptr<kBf16>(f.p1, s.b, s.r, is_target);
      const ChunkSpan<kBf16> sp(rp, f.p1.V, s.chunk, f.p1.nc);
      const uint32_t bytes = sp.bytes();
      if (bytes) {
        fence_proxy_async_smem();  // the stage was last read through the generic proxy
        mbar_expect_tx(full, bytes);
        bulk_load(stage, sp.body(rp), bytes, full);
        return;
      }
    }
  }
  mbar_arrive(full);
}

template <bool kBf16>
__device__ __forceinline__ bool pass1_staged(const FusedParams& f, const StagePlan& s,
                                             const uint4* sm, RowAcc* scratch) {
  const Pass1Params& p = f.p1;
  bool is_target;
  const char* rp = row_ptr<kBf16>(p, s.b, s.r, is_target);
  RowAcc a{-INFINITY, 0.0f, 0x7fffffff, 0};
  if (s.mode != kRowSkip) {
    const ChunkSpan<kBf16> sp(rp, p.V, s.chunk, p.nc);
    if (s.mode == kRowLse) {
      const float c = __fdiv_rn(kLog2e, __ldg(p.temps + s.b));
      scan_staged<kBf16, kRowLse, kConsumers>(a, rp, p.V, s.chunk, p.nc, sp, sm, c);
      a = block_reduce_acc<kRowLse, kConsumers>(a, c, scratch);
    } else {
      scan_staged<kBf16, kRowArgmax, kConsumers>(a, rp, p.V, s.chunk, p.nc, sp, sm, 0.0f);
      a = block_reduce_acc<kRowArgmax, kConsumers>(a, 0.0f, scratch);
    }
  }
  return publish_partial<kConsumers>(p, s.b, s.r, s.chunk, a);
}

template <bool kBf16>
__global__ void __launch_bounds__(kFusedThreads, 2) fused_single_kernel(FusedParams f) {
  extern __shared__ __align__(128) uint4 stage[];  // kStages x kStageBytes
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ long long slot[kStages];
  __shared__ RowAcc rows[kMaxRowsPerSeq];
  __shared__ RowAcc scratch[kConsumers / 32];
  __shared__ float4 race_scratch[kConsumers / 32];
  __shared__ unsigned s_flag;
  __shared__ int s_last;
  __shared__ volatile int s_abort;
  // Wait for the previous grid in the stream (programmatic dependent launch),
  // then let the next one start launching its CTAs.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const long long total = f.n1 + f.n2;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  if (tid >= kConsumers) {
    // ---- producer warp (one lane) ----
    if (tid == kConsumers) {
      uint32_t emask = (1u << kStages) - 1;  // a fresh barrier's "previous" phase is complete
      for (int s = 0;; s = (s + 1) % kStages) {
        if (s_abort || !mbar_wait(&empty[s], (emask >> s) & 1u, f.error)) {
          s_abort = 1;
          slot[s] = total;  // let the consumers stop
          mbar_arrive(&full[s]);
          break;
        }
        emask ^= 1u << s;
        const long long q = static_cast<long long>(atomicAdd(f.head, 1ull));
        slot[s] = q;
        produce<kBf16>(f, q, total, stage + static_cast<size_t>(s) * (kStageBytes / 16), &full[s]);
        if (q >= total) break;
      }
    }
    return;
  }

  // ---- consumer warps ----
  uint32_t fmask = 0u;
  for (int s = 0;; s = (s + 1) % kStages) {
    if (tid == 0 && !mbar_wait(&full[s], (fmask >> s) & 1u, f.error)) s_abort = 1;
    block_sync<kConsumers>();
    if (s_abort) break;
    mbar_try_wait(&full[s], (fmask >> s) & 1u);  // acquire the stage in every consumer
    fmask ^= 1u << s;
    const long long q = slot[s];
    if (q >= total) break;
    const StagePlan pl = plan_item<kBf16>(f, q);
    if (pl.r >= 0) {
      if (pass1_staged<kBf16>(f, pl, stage + static_cast<size_t>(s) * (kStageBytes / 16), scratch)) {
        combine_rows<kConsumers>(f.p1, pl.b, rows);
        if (tid < 32) decide_single<kBf16>(f.p1, pl.b, rows);
      }
    } else {
      pass2_item<kBf16>(f, pl.b, pl.chunk, race_scratch, &s_flag, &s_last);
    }
    block_sync<kConsumers>();  // every consumer is done with stage s
    if (tid == 0) mbar_arrive(&empty[s]);
  }
  if (tid == 0) {
    const unsigned n = atomicAdd(f.exited, 1u);
    if (n == gridDim.x - 1) {  // last CTA out leaves the queue reset
      *f.head = 0ull;
      *f.exited = 0u;
    }
  }
}

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
  p1.nc = lay.nc;
  p1.rps = 2 * gamma + 1;
  p1.seed = seed;
  p1.step = static_cast<uint32_t>(step);
  p1.part = reinterpret_cast<RowPartial*>(ws + lay.part1);
  p1.ticket = reinterpret_cast<unsigned*>(ws + lay.ticket1);
  p1.rowstat = nullptr;
  p1.info = reinterpret_cast<SeqInfo*>(ws + lay.info);
  p1.flag = reinterpret_cast<unsigned*>(ws + lay.flag);
  p1.accept_len = out_accept_len;
  p1.out_tokens = out_tokens;
  p1.out_lp = out_lp;
  p1.out_lq = out_lq;
  Pass2Params& p2 = f.p2;
  p2.target = target;
  p2.draft = draft;
  p2.B = B;
  p2.gamma = gamma;
  p2.V = V;
  p2.nc2 = lay.nc2;
  p2.blocks_per_chunk = ((V + 3) / 4 + lay.nc2 - 1) / lay.nc2;
  p2.seed = seed;
  p2.step = static_cast<uint32_t>(step);
  p2.info = p1.info;
  p2.part = reinterpret_cast<RacePartial*>(ws + lay.part2);
  p2.ticket = reinterpret_cast<unsigned*>(ws + lay.ticket2);
  p2.out_tokens = out_tokens;
  f.head = reinterpret_cast<unsigned long long*>(ws + lay.ctl);
  f.exited = reinterpret_cast<unsigned*>(ws + lay.ctl + 8);
  f.error = reinterpret_cast<unsigned*>(ws + lay.ctl + 12);
  f.a = p1.rps * p1.nc;
  f.n1 = static_cast<long long>(B) * f.a;
  f.n2 = static_cast<long long>(B) * lay.nc2;
  const bool bf16 = dtype == SV_BF16;
  const int S = resident_ctas(bf16);
  const long long items = f.n1 + f.n2;
  const unsigned grid = static_cast<unsigned>(items < S ? items : S);
  // Pass-2 items of a sequence are queued about one resident wave of items
  // (every CTA's stages plus the one in hand) after its pass-1 items, so its
  // decision is usually made before they are taken.
  const long long inflight = static_cast<long long>(grid) * (kStages + 1);
  const long long lag = inflight / f.a + 1;
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
