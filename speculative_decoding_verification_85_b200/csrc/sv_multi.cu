// sv_multi.cu -- multi-draft verification, "SpecTr-GBV: Multi-Draft Block
// Verification Accelerating Speculative Decoding", Methodology, Algorithm 1.
//
// One thread-block cluster of kC CTAs per sequence (16 when the batch's
// clusters fit in one wave, else 8); CTA `rank` owns the
// vocabulary slice [rank * slice, (rank + 1) * slice).  Every V-wide quantity
// of the algorithm is a sum (or a race) over the slices: each CTA reduces its
// slice, writes its partial into every CTA's exchange buffer through
// distributed shared memory, and after one cluster barrier every CTA adds the
// kC partials in rank order -- so every CTA holds the same value and takes
// the same decisions, with no further communication.  The steps:
//   1. row statistics (maximum, softmax sum, first argmax) of the L + 1 target
//      and L draft rows (one exchange);
//   2. the residual law R = P_0 and its sum (one exchange);
//   3. per draft k, in index order: the sub-block weights w_i (scalars), all
//      sums A_i = sum_v max(w_i P_{i+1}(v) - Q_{i+1}(v), 0) of the draft in one
//      pass (one exchange), the acceptance coins h_i = A_i / (A_i + 1 - w_i)
//      (h_{L-1} = w_{L-1}) with the longest accepted sub-block kept, then the
//      update of R -- on an advance R <- norm(max(w P_tau - Q_tau, 0)), on a
//      rejection R <- norm(max(R - Q~, 0)) with Q~ the draft law at tau
//      conditioned on not being in the rejected set H (one exchange);
//   4. the correction token: an exponential race over R at tau, or over P_L
//      when the whole block was accepted (one exchange).
// When a slice's rows and R fit in shared memory they are staged there once
// (bulk copies); otherwise every pass reads them from global memory.
//
// Reading of the unprinted equations (as in the CPU definition): greedy
// block-verification weights; the longest accepted sub-block wins; on a
// rejection the draft law at tau is conditioned on not being in H.  A token in
// H has R = 0 after its rejection, so the residual update needs no membership
// test; H only decides which later drafts are skipped.
#include <cooperative_groups.h>

#include <atomic>
#include <climits>

#include "sv_cluster.cuh"
#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace cg = cooperative_groups;

namespace sv {

constexpr int kMdT = 512;                        // threads per CTA
constexpr int kMdW = kMdT / 32;
constexpr int kXBatch = 32;                      // row statistics per exchange
constexpr int kXSlot = 2 * kXBatch;              // doubles per rank in an exchange buffer
constexpr int kMaxStatRows = 256;                // row statistics per sequence (all row sets)
static_assert(SV_MAX_GAMMA <= kXSlot, "an exchange carries every A_i of a draft");

struct MdcParams {
  const void* target;  // [B][nsets][L + 1][V]
  const void* draft;   // [B][nsets][L][V]
  const int32_t* tokens;
  const float* temps;
  int B, K, L, V;
  int per_draft;    // 1: a row set per draft (nsets = K); 0: one shared set
  uint64_t seed;
  uint32_t step;
  int slice;        // vocabulary entries per CTA (a multiple of 8)
  int rowstride;    // bytes per staged row slice in shared memory (local variant)
  float* Rws;       // [B][2][V] residual laws in global memory (global variant)
  int32_t* accept_len;
  int32_t* out_tokens;
  int32_t* out_draft_index;
};

// Fixed part of the dynamic shared memory (the local variant adds the R
// buffers and the staged rows after it), for clusters of kC CTAs.
template <int kC>
struct alignas(16) MdSmem {
  double xb[2][kC][kXSlot];            // exchange buffers (written by every rank)
  float4 part[kMaxStatRows];           // this slice's row statistics
  double wred[kMdW][SV_MAX_GAMMA];     // per-warp partial sums
  double res[kXSlot];                  // results of the last exchange
  float m[kMaxStatRows];               // row maxima
  float is[kMaxStatRows];              // 1 / s, s = sum_v 2^{(z_v - m) c}
  int arg[kMaxStatRows];               // first argmax (greedy target rows)
  double w[SV_MAX_GAMMA];              // the current draft's sub-block weights
  double num[SV_MAX_GAMMA], den[SV_MAX_GAMMA];  // their step ratios
  int H[SV_MAX_DRAFTS];                // rejected tokens at tau
  float4 race[kMdW];
  const char* rowp[kMaxStatRows];      // this slice's entry 0 of row q (shared or global memory)
  uint64_t rbar[kMaxStatRows];         // staging barriers, one per row
  uint64_t xbar[2];                    // exchange barriers (one per exchange buffer)
  uint32_t xphase[2];                  // their current phase parity
  int xfail;                           // an exchange wait ran out of time
  double Rn, qH, keep, wbest;
  int tau, a, nH, skip, best, rcur;
};

template <int kC>
constexpr size_t md_fixed() {
  return (sizeof(MdSmem<kC>) + 127) / 128 * 128;
}

// The draft tokens' arrays follow the fixed part: [K][L] target / draft
// logits at the token (float2), tokens (int), sub-block acceptance uniforms
// (float); 16 bytes per draft token, rounded up to 128.
__host__ __device__ constexpr size_t md_token_bytes(int K, int L) {
  return (static_cast<size_t>(K) * L * 16 + 127) / 128 * 128;
}

// The kC partials of an exchange, in rank order: thread t < nv contributes
// `mine` as slot t of buffer `buf` to every CTA; once they have all arrived
// thread t adds slot t over the ranks into sm.res[t]; ends with a CTA barrier.
template <int kC, typename Cl>
__device__ __forceinline__ void exchange(Cl& cl, MdSmem<kC>& sm, int buf, int nv, double mine) {
  const int tid = threadIdx.x;
  const int rank = static_cast<int>(cl.block_rank());
  // every rank sends nv values to every rank: arm this CTA's barrier for them
  if (tid == 0) mbar_arrive_expect_tx(&sm.xbar[buf], static_cast<uint32_t>(nv * kC * sizeof(double)));
  if (tid < nv) {
    // the CTA's earlier shared-memory writes (R, read remotely later) are
    // ordered before the values that announce them (callers end with a CTA barrier)
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
    for (int q = 0; q < kC; ++q) st_async_f64(mapa(&sm.xb[buf][rank][tid], q), mine, mapa(&sm.xbar[buf], q));
  }
  if (!xbar_wait(&sm.xbar[buf], sm.xphase[buf])) sm.xfail = 1;
  if (tid < nv) {
    double s = 0.0;
    for (int q = 0; q < kC; ++q) s += sm.xb[buf][q][tid];
    sm.res[tid] = s;
  }
  __syncthreads();
  if (tid == 0) sm.xphase[buf] ^= 1u;
  __syncthreads();
}

// One value slot v of a CTA-wide sum: each warp's total lands in sm.wred[warp][v].
template <int kC>
__device__ __forceinline__ void warp_sum_to(MdSmem<kC>& sm, int v, double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_down_sync(0xffffffffu, x, off);
  if ((threadIdx.x & 31) == 0) sm.wred[threadIdx.x >> 5][v] = x;
}

__device__ __forceinline__ double step_weight(double w, double num, double den) {
  if (den > 0.0) {
    const double t = w * (num / den);
    return t < 1.0 ? t : 1.0;
  }
  return (w > 0.0 && num > 0.0) ? 1.0 : 0.0;
}

template <bool kBf16, bool kLocal, int kC>
__global__ void __launch_bounds__(kMdT) md_cluster_kernel(const __grid_constant__ MdcParams p) {
  constexpr size_t es = kBf16 ? 2 : 4;
  extern __shared__ __align__(128) char dyn[];
  MdSmem<kC>& sm = *reinterpret_cast<MdSmem<kC>*>(dyn);
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int b = blockIdx.x / kC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, L = p.L, V = p.V, rps = 2 * L + 1;
  const int nsets = p.per_draft ? K : 1;
  const int v0 = rank * p.slice;
  const int n = max(0, min(V - v0, p.slice));  // entries of this slice
  // the rows, numbered q = set * rps + r: per row set the target rows 0..L,
  // then the draft rows 0..L-1 as r = L+1..2L.  All of them are staged at
  // once, before the temperature is known; a greedy sequence reads only its
  // target rows.
  const int nrows = rps;
  const int nq = nsets * nrows;
  const size_t rowb = static_cast<size_t>(V) * es;
  const char* tgt = static_cast<const char*>(p.target) + static_cast<size_t>(b) * nsets * (L + 1) * rowb;
  const char* drf = static_cast<const char*>(p.draft) + static_cast<size_t>(b) * nsets * L * rowb;
  auto grow = [&](int q) -> const char* {  // global row q
    const int set = q / nrows, r = q - set * nrows;
    return r <= L ? tgt + (static_cast<size_t>(set) * (L + 1) + r) * rowb
                  : drf + (static_cast<size_t>(set) * L + (r - L - 1)) * rowb;
  };
  auto qt = [&](int set, int i) { return set * nrows + i; };          // target row i of a set
  auto qd = [&](int set, int i) { return set * nrows + L + 1 + i; };  // draft row i of a set
  char* const tokreg = dyn + md_fixed<kC>();
  float2* const s_zg = reinterpret_cast<float2*>(tokreg);
  int* const s_tok = reinterpret_cast<int*>(tokreg + static_cast<size_t>(K) * L * sizeof(float2));
  float* const s_eta = reinterpret_cast<float*>(tokreg + static_cast<size_t>(K) * L * (sizeof(float2) + sizeof(int)));
  char* const dynrest = tokreg + md_token_bytes(K, L);
  float* Rb[2];
  char* srows = nullptr;
  if constexpr (kLocal) {
    Rb[0] = reinterpret_cast<float*>(dynrest);
    Rb[1] = Rb[0] + p.slice;
    srows = dynrest + 2 * static_cast<size_t>(p.slice) * sizeof(float);
  } else {
    Rb[0] = p.Rws + static_cast<size_t>(b) * 2 * V + v0;
    Rb[1] = Rb[0] + V;
  }
  // logit e (0 <= e < n) of a row slice that starts at rp (shared memory when
  // staged, else global memory)
  auto zat = [&](const char* rp, int e) -> float {
    if constexpr (kLocal) {
      if constexpr (kBf16)
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(rp)[e]) << 16);
      else
        return reinterpret_cast<const float*>(rp)[e];
    } else {
      return logit_at<kBf16>(rp, e);
    }
  };
  for (int q = tid; q < nq; q += kMdT) {
    const char* g = grow(q) + static_cast<size_t>(v0) * es;
    sm.rowp[q] = kLocal ? srows + static_cast<size_t>(q) * p.rowstride + (reinterpret_cast<uintptr_t>(g) & 15u)
                        : g;
  }
  auto zrow = [&](int q, int e) -> float { return zat(sm.rowp[q], e); };

  // ---- staging of the slice's rows (a bulk copy and a barrier per row;
  // rows start at the same offset modulo 16 in shared and in global memory,
  // so the aligned body of each row slice is one bulk copy), then the draft
  // tokens, their logits and the sub-block acceptance uniforms while the
  // rows are in flight
  if (tid == 0) {
    if (kLocal)
      for (int q = 0; q < nq; ++q) mbar_init(&sm.rbar[q], 1);
    mbar_init(&sm.xbar[0], 1);
    mbar_init(&sm.xbar[1], 1);
    sm.xphase[0] = sm.xphase[1] = 0u;
    sm.xfail = 0;
    mbar_init_fence();
  }
  __syncthreads();  // the barriers are initialised before any thread waits on them
  bool scalar_copies = false;
  if constexpr (kLocal) scalar_copies = stage_rows_issue<es, kMdT>(grow, nq, v0, n, srows, p.rowstride, sm.rbar);
  const float T = __ldg(p.temps + b);
  const bool tvalid = (T >= 0.0f) && !isinf(T);
  const bool greedy = tvalid && T == 0.0f;
  auto needed = [&](int q) { return !greedy || q % rps <= L; };  // rows the sequence reads
  // every staged row has landed before the CTA leaves (rows a greedy sequence
  // never read included)
  auto drain = [&]() {
    if constexpr (kLocal)
      if (tid == 0)
        for (int q = 0; q < nq; ++q) (void)mbar_wait(&sm.rbar[q], 0);
  };
  // every CTA's barriers are initialised before any remote store: arrive
  // now, wait just before the first exchange
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  // draft token t of the sequence ([K][L] order): the token, its two logits
  // and its sub-block acceptance uniform ((x >> 8) 2^-24, exact in fp32)
  auto token_info = [&](int t, int& x, float2& z, float& u) {
    x = __ldg(p.tokens + static_cast<size_t>(b) * K * L + t);
    const int k = t / L, i = t - k * L, set = p.per_draft ? k : 0;
    z = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    if (tvalid && !greedy && x >= 0 && x < V) {
      z.x = logit_at<kBf16>(grow(qt(set, i)), x);
      z.y = logit_at<kBf16>(grow(qd(set, i)), x);
    }
    u = static_cast<float>(accept_uniform(keyed_block(p.seed, p.step, kTagMdEta, b, k, i, i).x));
  };
  // the first kMdT tokens, by the highest threads (whose warps have no row
  // when the rows are fewer than the warps): loaded now, stored after the
  // row statistics
  const int tt = kMdT - 1 - tid;
  int x0 = 0;
  float2 z0 = make_float2(0.0f, 0.0f);
  float u0 = 0.0f;
  if (tt < K * L) token_info(tt, x0, z0, u0);
  if (scalar_copies) __syncthreads();  // the scalar head and tail copies

  // ---- 1. row statistics of the slice: a warp per row (q = warp, warp +
  // kMdW, ...; lane l takes entries l, l + 32, ...) as soon as the row has
  // landed: the maximum (NaN-propagating; for greedy rows with its first
  // index), then the scaled sum s = sum_v 2^{(z_v - m) c} against it, each
  // with four independent chains; then one exchange per batch of rows,
  // merged in rank order
  int buf = 0;
  bool row_ok = true;
  {
    const float c = tvalid && !greedy ? __fdiv_rn(kLog2e, T) : 0.0f;
    float4* part = sm.part;  // [nq] this slice's row statistics
    for (int q = warp; q < nq; q += kMdW) {
      bool landed = true;
      if constexpr (kLocal) landed = mbar_wait(&sm.rbar[q], 0);
      if (!needed(q)) {
        if (lane == 0) part[q] = make_float4(-INFINITY, 0.0f, __int_as_float(0x7fffffff), __int_as_float(0));
        continue;
      }
      const char* gq = grow(q) + static_cast<size_t>(v0) * es;
      const char* rp = kLocal ? srows + static_cast<size_t>(q) * p.rowstride + (reinterpret_cast<uintptr_t>(gq) & 15u) : gq;
      float m = -INFINITY, sum = 0.0f;
      int arg = 0x7fffffff, bad = landed ? 0 : 1;
      if (tvalid && landed) {
        if (greedy) {
          for (int e = lane; e < n; e += 32) {
            const float z = zat(rp, e);
            if (z != z) bad = 1;
            else if (z > m) {
              m = z;
              arg = v0 + e;
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
            const int a2 = __shfl_xor_sync(0xffffffffu, arg, off);
            argmax_merge(m, arg, m2, a2);
          }
        } else {
          float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          for (int e0 = lane; e0 < n; e0 += 128)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              if (e0 + 32 * k < n) mk[k] = max_nan(mk[k], zat(rp, e0 + 32 * k));
          m = max_nan(max_nan(mk[0], mk[1]), max_nan(mk[2], mk[3]));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
          if (m != m) {
            bad = 1;
          } else if (m != -INFINITY) {
            float sk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int e0 = lane; e0 < n; e0 += 128)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                if (e0 + 32 * k < n) sk[k] += ex2_approx((zat(rp, e0 + 32 * k) - m) * c);
            sum = (sk[0] + sk[1]) + (sk[2] + sk[3]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
          }
        }
        bad = __any_sync(0xffffffffu, bad) ? 1 : 0;
      }
      if (lane == 0) part[q] = make_float4(m, sum, __int_as_float(arg), __int_as_float(bad));
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    for (int q0 = 0; q0 < nq; q0 += kXBatch) {
      const int nb = min(kXBatch, nq - q0);
      if (tid == 0) mbar_arrive_expect_tx(&sm.xbar[buf], static_cast<uint32_t>(nb * kC * sizeof(float4)));
      if (tid < nb) {
        const float4 v = part[q0 + tid];
        for (int r = 0; r < kC; ++r)
          st_async_f4(mapa(&sm.xb[buf][rank][2 * tid], r), v, mapa(&sm.xbar[buf], r));
      }
      if (!xbar_wait(&sm.xbar[buf], sm.xphase[buf])) sm.xfail = 1;
      if (tid < nb) {
        RowAcc a{-INFINITY, 0.0f, 0x7fffffff, 0};
        for (int r = 0; r < kC; ++r) {
          const float4 x = *reinterpret_cast<const float4*>(&sm.xb[buf][r][2 * tid]);
          const RowAcc o{x.x, x.y, __float_as_int(x.z), __float_as_int(x.w)};
          if (greedy) acc_merge<kRowArgmax>(a, o, c); else acc_merge<kRowLse>(a, o, c);
        }
        const int q = q0 + tid;
        sm.m[q] = a.m;
        sm.is[q] = greedy ? 0.0f : 1.0f / a.s;
        sm.arg[q] = a.arg;
        bool rv = !a.bad && isfinite(a.m);
        if (!greedy) rv = rv && isfinite(__fdiv_rn(a.m, T));
        if (needed(q)) row_ok = row_ok && rv;
      }
      __syncthreads();  // every thread has read the buffer
      if (tid == 0) sm.xphase[buf] ^= 1u;
      buf ^= 1;
      __syncthreads();
    }
  }
  if (tt < K * L) {
    s_tok[tt] = x0;
    s_zg[tt] = z0;
    s_eta[tt] = u0;
  }
  for (int t = kMdT + tid; t < K * L; t += kMdT) {  // more than kMdT draft tokens
    int x;
    float2 z;
    float u;
    token_info(t, x, z, u);
    s_tok[t] = x;
    s_zg[t] = z;
    s_eta[t] = u;
  }
  __syncthreads();
  // validity: temperature, rows, tokens (the same in every CTA of the cluster)
  bool ok = tvalid && row_ok && !sm.xfail;
  for (int t = tid; t < K * L; t += kMdT) ok = ok && s_tok[t] >= 0 && s_tok[t] < V;
  ok = __syncthreads_and(ok);
  int32_t* tok = p.out_tokens + static_cast<size_t>(b) * (L + 1);
  if (!ok) {
    if (rank == 0) {
      for (int i = tid; i <= L; i += kMdT) tok[i] = -1;
      if (tid == 0) {
        p.accept_len[b] = -1;
        if (p.out_draft_index) p.out_draft_index[b] = -1;
      }
    }
    drain();
    cl.sync();  // every CTA returns here, after every remote store has landed
    return;
  }
  if (greedy) {
    // the accepted block is the longest draft prefix that matches the target
    // argmaxes of its row set (first draft on ties); the correction is the
    // argmax at tau of the accepted draft's rows (of row set 0 when nothing
    // was accepted: every draft shares the empty prefix)
    if (rank == 0 && tid == 0) {
      int tau = 0, a = -1;
      for (int k = 0; k < K; ++k) {
        const int set = p.per_draft ? k : 0;
        int m = 0;
        while (m < L && s_tok[k * L + m] == sm.arg[qt(set, m)]) ++m;
        if (m > tau) {
          tau = m;
          a = k;
        }
      }
      const int sa = p.per_draft && a >= 0 ? a : 0;
      for (int i = 0; i <= L; ++i)
        tok[i] = i < tau ? s_tok[a * L + i] : (i == tau ? sm.arg[qt(sa, tau)] : -1);
      p.accept_len[b] = tau;
      if (p.out_draft_index) p.out_draft_index[b] = a;
    }
    drain();
    cl.sync();
    return;
  }

  // P and Q of row q at entry e: 2^{(z - m_q) c} / s_q with c = log2(e) / T, the
  // same MUFU exponential that built the row sums (each law sums to 1 to
  // within its 2^-22 relative error); one subtraction, one multiply, one ex2
  // and one multiply per value.
  const float cc = __fdiv_rn(kLog2e, T);
  struct Law {
    const char* rp;
    float m, is;
  };
  auto law = [&](int q) { return Law{sm.rowp[q], sm.m[q], sm.is[q]}; };
  auto at = [&](const Law& l, int e) -> float { return ex2_approx((zat(l.rp, e) - l.m) * cc) * l.is; };
  auto prob = [&](int q, int e) -> float { return at(law(q), e); };
  auto prob_x = [&](int q, float z) -> float { return ex2_approx((z - sm.m[q]) * cc) * sm.is[q]; };
  auto exch1 = [&](double x) {  // one value: CTA sum, then cluster sum into sm.res[0]
    warp_sum_to(sm, 0, x);
    __syncthreads();
    double loc = 0.0;
    if (tid == 0)
      for (int w = 0; w < kMdW; ++w) loc += sm.wred[w][0];
    exchange(cl, sm, buf, 1, loc);
    buf ^= 1;
  };

  // ---- 2. R <- P_0 (row set 0: every draft shares the empty prefix)
  {
    double loc = 0.0;
    for (int e = tid; e < n; e += kMdT) {
      const float pv = prob(qt(0, 0), e);
      Rb[0][e] = pv;
      loc += pv;
    }
    exch1(loc);
    if (tid == 0) {
      sm.Rn = sm.res[0];
      sm.tau = 0;
      sm.a = -1;
      sm.nH = 0;
      sm.qH = 0.0;
      sm.rcur = 0;
    }
    __syncthreads();
  }

  // ---- 3. the drafts in index order
  for (int k = 0; k < K; ++k) {
    const int set = p.per_draft ? k : 0;
    if (warp == 0) {
      // lane 0: whether the draft is considered; then lane r the ratio
      // num / den of position tau + r (and + 32), in parallel; then lane 0
      // the weights w_i in order
      const int tau = sm.tau;
      const int* x = s_tok + k * L;
      int skip = 0;
      if (lane == 0) {
        skip = tau == L ? 2 : 0;
        if (!skip && tau > 0) {
          const int* xa = s_tok + sm.a * L;
          for (int i = 0; i < tau; ++i)
            if (x[i] != xa[i]) skip = 1;
        }
        if (!skip)
          for (int h = 0; h < sm.nH; ++h)
            if (sm.H[h] == x[tau]) skip = 1;
        sm.skip = skip;
      }
      skip = __shfl_sync(0xffffffffu, skip, 0);
      if (!skip) {
        const double keep = 1.0 - sm.qH;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int i = tau + lane + 32 * h2;
          if (i < L) {
            double num, den;
            if (i == tau) {
              // R at the draft's token: read from the CTA that owns that entry
              const int xt = x[tau], owner = xt / p.slice, eo = xt - owner * p.slice;
              float rx;
              if constexpr (kLocal) {
                const float* Rl = reinterpret_cast<const float*>(dynrest) + sm.rcur * p.slice;
                rx = cl.map_shared_rank(Rl, owner)[eo];
              } else {
                rx = p.Rws[static_cast<size_t>(b) * 2 * V + static_cast<size_t>(sm.rcur) * V + xt];
                (void)eo;
              }
              num = static_cast<double>(rx) / sm.Rn;
              den = keep > 0.0 ? static_cast<double>(prob_x(qd(set, tau), s_zg[k * L + tau].y)) / keep : 0.0;
            } else {
              num = prob_x(qt(set, i), s_zg[k * L + i].x);
              den = prob_x(qd(set, i), s_zg[k * L + i].y);
            }
            sm.num[i] = num;
            sm.den[i] = den;
          }
        }
        __syncwarp();
        if (lane == 0) {
          sm.keep = keep;
          double w = 1.0;
          for (int i = tau; i < L; ++i) {
            w = step_weight(w, sm.num[i], sm.den[i]);
            sm.w[i] = w;
          }
        }
      }
    }
    __syncthreads();
    if (sm.skip == 2) break;
    if (sm.skip) continue;
    const int tau = sm.tau;
    const int* x = s_tok + k * L;
    // all of the draft's sums A_i, i = tau .. L-2, in one pass (at least one
    // exchange, which also orders the R reads above before any R update)
    const int nA = max(L - 1 - tau, 0);
    for (int i = tau; i < L - 1; ++i) {
      const float wf = static_cast<float>(sm.w[i]);
      const Law lp = law(qt(set, i + 1)), lq = law(qd(set, i + 1));
      double loc = 0.0;
      for (int e = tid; e < n; e += kMdT) {
        const float t = wf * at(lp, e) - at(lq, e);
        if (t > 0.0f) loc += t;
      }
      warp_sum_to(sm, i - tau, loc);
    }
    __syncthreads();
    {
      double loc = 0.0;
      if (tid < nA)
        for (int w = 0; w < kMdW; ++w) loc += sm.wred[w][tid];
      exchange(cl, sm, buf, max(nA, 1), loc);
      buf ^= 1;
    }
    if (warp == 0) {
      // the coins h_i, lane r for position tau + r (and + 32); the accepted
      // sub-block is the longest one: up to the last position whose coin
      // came up
      unsigned acc[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int i = tau + lane + 32 * h2;
        bool up = false;
        if (i < L) {
          const double w = sm.w[i];
          double h;
          if (i < L - 1) {
            const double A = sm.res[i - tau];
            const double den = A + 1.0 - w;
            h = den == 0.0 ? 1.0 : A / den;
          } else {
            h = w;
          }
          up = static_cast<double>(s_eta[k * L + i]) < h;
        }
        acc[h2] = __ballot_sync(0xffffffffu, up);
      }
      if (lane == 0) {
        int best = tau;
        double wbest = 1.0;
        const int r = acc[1] ? 63 - __clz(acc[1]) : (acc[0] ? 31 - __clz(acc[0]) : -1);
        if (r >= 0) {
          best = tau + r + 1;
          wbest = sm.w[tau + r];
        }
        sm.best = best;
        sm.wbest = wbest;
      }
    }
    __syncthreads();
    const int best = sm.best;
    const int rc = sm.rcur;
    float* Rcur = Rb[rc];
    float* Rnew = Rb[rc ^ 1];
    if (best > tau) {
      if (best < L) {
        const float wb = static_cast<float>(sm.wbest);
        const Law lp = law(qt(set, best)), lq = law(qd(set, best));
        double loc = 0.0;
        for (int e = tid; e < n; e += kMdT) {
          const float t = wb * at(lp, e) - at(lq, e);
          const float rv = t > 0.0f ? t : 0.0f;
          Rnew[e] = rv;
          loc += rv;
        }
        exch1(loc);
        if (sm.res[0] > 0.0) {
          if (tid == 0) sm.Rn = sm.res[0];
        } else {
          // the residual vanished: the correction law is P_tau itself
          double l2 = 0.0;
          for (int e = tid; e < n; e += kMdT) {
            const float pv = prob(qt(set, best), e);
            Rnew[e] = pv;
            l2 += pv;
          }
          exch1(l2);
          if (tid == 0) sm.Rn = sm.res[0];
        }
        if (tid == 0) sm.rcur = rc ^ 1;
      }
      if (tid == 0) {
        sm.tau = best;
        sm.a = k;
        sm.nH = 0;
        sm.qH = 0.0;
      }
    } else {
      const float inv_rn = static_cast<float>(1.0 / sm.Rn);
      const double keep = sm.keep;
      const float inv_keep = keep > 0.0 ? static_cast<float>(1.0 / keep) : 0.0f;
      const Law lq = law(qd(set, tau));
      double loc = 0.0;
      for (int e = tid; e < n; e += kMdT) {
        const float t = Rcur[e] * inv_rn - at(lq, e) * inv_keep;
        const float rv = t > 0.0f ? t : 0.0f;
        Rnew[e] = rv;
        loc += rv;
      }
      exch1(loc);
      if (tid == 0) {
        if (sm.res[0] > 0.0) {  // else R stays as it was (a vanished update changes nothing)
          sm.Rn = sm.res[0];
          sm.rcur = rc ^ 1;
        }
        sm.H[sm.nH++] = x[tau];
        sm.qH += static_cast<double>(prob_x(qd(set, tau), s_zg[k * L + tau].y));
      }
    }
    __syncthreads();
  }

  // ---- 4. correction token: race over P_L of the accepted draft's rows
  // (whole block accepted) or over R at tau
  const int tau = sm.tau;
  const int sa = p.per_draft && sm.a >= 0 ? sm.a : 0;
  const float* Rf = Rb[sm.rcur];
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
  const int g0 = v0 >> 2, g1 = (v0 + n + 3) >> 2;  // Philox blocks of the slice (v0 % 8 == 0)
  for (int g = g0 + tid; g < g1; g += kMdT) {
    const uint4 rnd = keyed_block(p.seed, p.step, kTagMdGumbel, b, 0, tau, static_cast<uint32_t>(g));
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int v = 4 * g + w, e = v - v0;
      if (e >= n) break;
      const float wt = tau == L ? prob(qt(sa, L), e) : Rf[e];
      if (!(wt > 0.0f)) continue;
      const float ev = exponential_from_bits(word_of(rnd, w));
      if (race_better(wt, ev, v, bw, be, bi)) {
        bw = wt;
        be = ev;
        bi = v;
      }
    }
  }
  race_reduce<kMdT>(bw, be, bi, sm.race);
  if (tid == 0)
    *reinterpret_cast<float4*>(cl.map_shared_rank(&sm.xb[buf][rank][0], 0)) =
        make_float4(bw, be, __int_as_float(bi), __int_as_float(sm.xfail));
  drain();
  cl.sync();
  if (rank == 0 && tid == 0) {
    bw = 0.0f;
    be = 1.0f;
    bi = INT_MAX;
    int fail = 0;
    for (int q = 0; q < kC; ++q) {
      const float4 g = *reinterpret_cast<const float4*>(&sm.xb[buf][q][0]);
      fail |= __float_as_int(g.w);
      if (race_better(g.x, g.y, __float_as_int(g.z), bw, be, bi)) {
        bw = g.x;
        be = g.y;
        bi = __float_as_int(g.z);
      }
    }
    if (fail) {  // an exchange wait of some rank ran out of time: no result
      for (int i = 0; i <= L; ++i) tok[i] = -1;
      p.accept_len[b] = -1;
      if (p.out_draft_index) p.out_draft_index[b] = -1;
      return;
    }
    const int a = sm.a;
    for (int i = 0; i <= L; ++i) tok[i] = i < tau ? s_tok[a * L + i] : (i == tau ? bi : -1);
    p.accept_len[b] = tau;
    if (p.out_draft_index) p.out_draft_index[b] = a;
  }
}

// ------------------------------------------------------------------ launch
namespace {
constexpr size_t kMaxDynSmem = 227 * 1024;

struct MdShape {
  int slice, rowstride;
  size_t smem_local;
};

MdShape md_shape(int rows, int V, int dtype, int C, size_t fixed) {
  const size_t es = dtype == SV_BF16 ? 2 : 4;
  MdShape s{};
  s.slice = ((V + C - 1) / C + 7) / 8 * 8;
  s.rowstride = static_cast<int>((static_cast<size_t>(s.slice) * es + 16 + 15) / 16 * 16);
  s.smem_local = fixed + 2 * static_cast<size_t>(s.slice) * sizeof(float) +
                 static_cast<size_t>(rows) * s.rowstride;
  return s;
}

template <int kC, typename Kernel>
cudaLaunchConfig_t md_config(Kernel, int B, size_t smem, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(B) * kC);
  cfg.blockDim = dim3(kMdT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Clusters of a variant that can be resident at once at this shared-memory
// size (the variant opted into the largest size and, for 16 CTAs, into a
// non-portable cluster size); 0 if none.
template <int kC, typename Kernel>
int md_clusters(Kernel kernel, size_t smem) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxDynSmem)) != cudaSuccess ||
      (kC > 8 && cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)) {
    (void)cudaGetLastError();
    return 0;
  }
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = md_config<kC>(kernel, 1, smem, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

// md_clusters asked once per device, variant and size (rounded up to 8 KB).
template <bool kBf16, bool kLocal, int kC>
int md_capacity(size_t smem) {
  constexpr size_t kStep = 8 * 1024;
  constexpr int kClasses = static_cast<int>((kMaxDynSmem + kStep - 1) / kStep) + 1;
  static std::atomic<int> cap[kClasses][64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int cls = static_cast<int>((smem + kStep - 1) / kStep);
  if (cls >= kClasses) return 0;
  int v = cap[cls][dev].load(std::memory_order_relaxed);
  if (v == 0) {
    const size_t probe = static_cast<size_t>(cls) * kStep < kMaxDynSmem ? static_cast<size_t>(cls) * kStep : kMaxDynSmem;
    const int n = md_clusters<kC>(md_cluster_kernel<kBf16, kLocal, kC>, probe);
    v = n > 0 ? n : -1;
    cap[cls][dev].store(v, std::memory_order_relaxed);
  }
  return v > 0 ? v : 0;
}

// Launch with clusters of kC CTAs: the variant that stages the rows in
// shared memory when they fit, else the one that reads them from global
// memory.  With need_wave, only when all B clusters fit in one wave.  Sets
// `launched`; returns a status.
template <bool kBf16, int kC>
int md_try(MdcParams p, int B, int rows, bool need_wave, cudaStream_t stream, bool& launched) {
  launched = false;
  const size_t fixed = md_fixed<kC>() + md_token_bytes(p.K, p.L);
  const MdShape sh = md_shape(rows, p.V, kBf16 ? SV_BF16 : SV_F32, kC, fixed);
  p.slice = sh.slice;
  p.rowstride = sh.rowstride;
  const bool local = sh.smem_local <= kMaxDynSmem && md_capacity<kBf16, true, kC>(sh.smem_local) > 0;
  const size_t smem = local ? sh.smem_local : fixed;
  const int cap = local ? md_capacity<kBf16, true, kC>(smem) : md_capacity<kBf16, false, kC>(smem);
  if (cap <= 0 || (need_wave && B > cap)) return SV_OK;
  cudaLaunchAttribute attr[1];
  cudaError_t e;
  if (local) {
    const cudaLaunchConfig_t cfg = md_config<kC>(md_cluster_kernel<kBf16, true, kC>, B, smem, stream, attr);
    e = cudaLaunchKernelEx(&cfg, md_cluster_kernel<kBf16, true, kC>, p);
  } else {
    const cudaLaunchConfig_t cfg = md_config<kC>(md_cluster_kernel<kBf16, false, kC>, B, smem, stream, attr);
    e = cudaLaunchKernelEx(&cfg, md_cluster_kernel<kBf16, false, kC>, p);
  }
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "multi-draft kernel launch failed: %s", cudaGetErrorString(e));
  launched = true;
  return SV_OK;
}
}  // namespace

size_t multidraft_global_bytes(int B, int V) {  // residual laws of the global variant
  return 2 * static_cast<size_t>(B) * static_cast<size_t>(V) * sizeof(float);
}

int multidraft_max_row_sets(int L) { return kMaxStatRows / (2 * L + 1); }

int launch_multi(const void* target, const void* draft, const int32_t* tokens,
                 const float* temps, int B, int K, int L, int V, int dtype, int per_draft,
                 uint64_t seed, uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                 int32_t* out_draft_index, void* workspace, const Layout& lay,
                 cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  const int nsets = per_draft ? K : 1;
  if (nsets * (2 * L + 1) > kMaxStatRows)
    return set_error(SV_ERR_UNSUPPORTED,
                     "per-draft rows: K (2L + 1) = %d row statistics per sequence, more than %d",
                     nsets * (2 * L + 1), kMaxStatRows);
  MdcParams p{};
  p.target = target;
  p.draft = draft;
  p.tokens = tokens;
  p.temps = temps;
  p.B = B;
  p.K = K;
  p.L = L;
  p.V = V;
  p.per_draft = per_draft ? 1 : 0;
  p.seed = seed;
  p.step = static_cast<uint32_t>(step);
  p.Rws = reinterpret_cast<float*>(ws + lay.resid);
  p.accept_len = out_accept_len;
  p.out_tokens = out_tokens;
  p.out_draft_index = out_draft_index;
  if (static_cast<long long>(B) * 16 > INT_MAX)
    return set_error(SV_ERR_INVALID_ARG, "B too large for one launch");
  // Clusters of 16 CTAs when all B of them fit in one wave (each CTA then
  // stages and sweeps half as many entries), else of 8.
  const int rows = nsets * (2 * L + 1);
  const bool bf16 = dtype == SV_BF16;
  bool launched = false;
  int st = bf16 ? md_try<true, 16>(p, B, rows, true, stream, launched)
                : md_try<false, 16>(p, B, rows, true, stream, launched);
  if (st == SV_OK && !launched)
    st = bf16 ? md_try<true, 8>(p, B, rows, false, stream, launched)
              : md_try<false, 8>(p, B, rows, false, stream, launched);
  if (st != SV_OK) return st;
  if (!launched) return set_error(SV_ERR_CUDA, "multi-draft cluster kernel cannot be made resident");
  return check_launch("multidraft");
}

}  // namespace sv
