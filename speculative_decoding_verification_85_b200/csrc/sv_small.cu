// sv_small.cu -- single-draft verification of small batches: one
// thread-block cluster of kSdC CTAs per sequence, everything on chip.
//
// The same verification as the row and draw kernels (FlashSpec, Methodology
// s.1; FlexDraft, Problem definition; Speculative Speculative Decoding, s.2
// Saguaro sampling), with the latency of a small batch in mind: CTA `rank`
// stages its vocabulary slice of every row the sequence needs into shared
// memory once (bulk copies), and the cross-slice steps are exchanges of a few
// values through distributed shared memory instead of kernel boundaries:
//   1. row statistics of the slice (maximum, scaled softmax sum, first
//      argmax for greedy rows), exchanged and merged in rank order, so every
//      CTA holds the same row statistics;
//   2. every CTA takes the decision (one warp; only rank 0 writes it out);
//   3. level 1 of the draw race over the slice's race groups (slices are
//      whole groups of kRaceGroup entries), one exchange of the CTAs' best
//      groups, merged in rank order;
//   4. level 2 in the winning group by the CTA that holds it, which writes
//      the token.
// Used when one cluster per sequence fits in a wave, the slices of all rows
// fit in shared memory and a slice has at most 4096 entries; other shapes
// take the streaming kernels.
#include <cooperative_groups.h>

#include <atomic>
#include <climits>

#include "sv_cluster.cuh"
#include "sv_decide.cuh"
#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace cg = cooperative_groups;

namespace sv {

constexpr int kSdC = 8;      // CTAs per cluster (one sequence)
constexpr int kSdT = 512;    // threads per CTA
constexpr int kSdW = kSdT / 32;
constexpr int kSdBatch = 32; // row statistics per exchange
static_assert(SV_MAX_GAMMA <= kSdT, "one thread per draft token");
constexpr int kSdMaxUnits = 64;               // level-1 work units (group parts) per slice
// Measured on a B200 (graph-replayed steps): for slices of up to 4096
// entries the cluster kernel is 6-11% faster than the row and draw kernels
// at B <= 8 and level at B = 16; for wider slices (V = 65536) it is slower.
constexpr int kSdMaxSlice = 4 * kRaceGroup;

struct SdParams {
  CallParams p;
  int slice;      // vocabulary entries per CTA (a multiple of kRaceGroup)
  int rowstride;  // bytes per staged row slice in shared memory
};

// Fixed part of the dynamic shared memory (the staged rows follow it).
struct alignas(16) SdSmem {
  float4 xb[2][kSdC][kSdBatch];      // exchange buffers (written by every rank)
  float4 part[kMaxRowsPerSeq];       // this slice's row statistics
  RowAcc rows[kMaxRowsPerSeq];       // merged row statistics (target rows, then draft rows)
  float gpart[kSdMaxUnits];          // race-group partial sums (level 1)
  float uacc[SV_MAX_GAMMA];          // acceptance uniforms ((x >> 8) 2^-24, exact in fp32)
  float gE[(SV_MAX_GAMMA + 1) * (kSdMaxSlice / kRaceGroup)];  // group exponentials [j][local group]
  float zsel[2 * SV_MAX_GAMMA];      // the draft tokens' target / draft logits
  int tok[SV_MAX_GAMMA];             // the draft tokens
  float4 race[kSdW];
  const char* rowp[kMaxRowsPerSeq];  // this slice's entry 0 of row q, in shared memory
  SeqInfo si;                        // the decision
  uint64_t rbar[kMaxRowsPerSeq];     // staging barriers, one per row
  uint64_t xbar[2];                  // exchange barriers (one per exchange buffer)
  uint32_t xphase[2];
  int xfail;                         // an exchange wait ran out of time
};

constexpr size_t kSdFixed = (sizeof(SdSmem) + 127) / 128 * 128;

// Every rank sends nv float4 values (thread t < nv sends `mine`) to slot
// [rank][t] of buffer `buf` on every rank, then waits (bounded) until all
// kSdC ranks' values have arrived here.  The caller reads sm.xb[buf] and then
// calls exchange_done.  A buffer is written again only two exchanges later,
// after every rank has sent the exchange in between, so every rank has read
// it by then.
template <typename Cl>
__device__ __forceinline__ void exchange_f4(Cl& cl, SdSmem& sm, int buf, int nv, float4 mine) {
  const int tid = threadIdx.x;
  const int rank = static_cast<int>(cl.block_rank());
  if (tid == 0) mbar_arrive_expect_tx(&sm.xbar[buf], static_cast<uint32_t>(nv * kSdC * sizeof(float4)));
  if (tid < nv) {
    // the values carry everything the receivers read: no fence needed
    for (int r = 0; r < kSdC; ++r) st_async_f4(mapa(&sm.xb[buf][rank][tid], r), mine, mapa(&sm.xbar[buf], r));
  }
  if (!xbar_wait(&sm.xbar[buf], sm.xphase[buf])) sm.xfail = 1;
}
__device__ __forceinline__ void exchange_done(SdSmem& sm, int& buf) {
  __syncthreads();  // every thread has read the buffer
  if (threadIdx.x == 0) sm.xphase[buf] ^= 1u;
  buf ^= 1;
  __syncthreads();
}

// Philox block (c0 = g) of the keyed counter (g, b, step, tag << 24 | j).
__device__ __forceinline__ uint4 sd_block(const CallParams& p, int b, uint32_t tag, int j, int g) {
  return keyed_block(p.seed, p.step, tag, static_cast<uint32_t>(b), 0, static_cast<uint32_t>(j),
                     static_cast<uint32_t>(g));
}

template <bool kBf16>
__global__ void __launch_bounds__(kSdT) sd_cluster_kernel(const __grid_constant__ SdParams f) {
  constexpr size_t es = kBf16 ? 2 : 4;
  extern __shared__ __align__(128) char dyn[];
  SdSmem& sm = *reinterpret_cast<SdSmem*>(dyn);
  char* srows = dyn + kSdFixed;
  cg::cluster_group cl = cg::this_cluster();
  const CallParams& p = f.p;
  const int rank = static_cast<int>(cl.block_rank());
  const int b = blockIdx.x / kSdC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = p.gamma, V = p.V;
  const int v0 = rank * f.slice;
  const int n = max(0, min(V - v0, f.slice));  // entries of this slice
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  // rows q = 0..g: target rows; q = g + 1 + i: draft row i.  All 2 gamma + 1
  // rows are staged at once, before the temperature is known (a greedy
  // sequence then reads only its target rows).
  const int nall = 2 * g + 1;
  const size_t rowb = static_cast<size_t>(V) * es;
  const char* tgt = static_cast<const char*>(p.target) + static_cast<size_t>(b) * (g + 1) * rowb;
  const char* drf = static_cast<const char*>(p.draft) + static_cast<size_t>(b) * g * rowb;
  auto grow = [&](int q) -> const char* {
    return q <= g ? tgt + static_cast<size_t>(q) * rowb : drf + static_cast<size_t>(q - g - 1) * rowb;
  };
  if (tid == 0) {
    for (int q = 0; q < nall; ++q) mbar_init(&sm.rbar[q], 1);
    mbar_init(&sm.xbar[0], 1);
    mbar_init(&sm.xbar[1], 1);
    sm.xphase[0] = sm.xphase[1] = 0u;
    sm.xfail = 0;
    mbar_init_fence();
  }
  __syncthreads();  // the barriers are initialised before any thread waits on them
  const bool scalar_copies = stage_rows_issue<es, kSdT>(grow, nall, v0, n, srows, f.rowstride, sm.rbar);
  // every CTA's barriers are initialised before any remote store: arrive
  // now, wait just before the first exchange
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  // the temperature and the draft tokens (draft token i by thread
  // kSdT - 1 - i, a warp without a row when the rows are fewer than the
  // warps), then the draft tokens' two logits: loads issued now, stored to
  // shared memory before the decision
  const float T = __ldg(p.temps + b);
  const int ti = kSdT - 1 - tid;  // this thread's draft token (if ti < gamma)
  int xi = 0;
  if (ti < g) xi = __ldg(p.tokens + static_cast<size_t>(b) * g + ti);
  const bool tvalid = (T >= 0.0f) && !isinf(T);
  const bool greedy = tvalid && T == 0.0f;
  const int nq = greedy ? g + 1 : nall;  // rows the sequence reads
  for (int q = tid; q < nall; q += kSdT) {
    const char* gp = grow(q) + static_cast<size_t>(v0) * es;
    sm.rowp[q] = srows + static_cast<size_t>(q) * f.rowstride + (reinterpret_cast<uintptr_t>(gp) & 15u);
  }
  auto zat = [&](const char* rp, int e) -> float {  // logit e (0 <= e < n) of a staged row slice
    if constexpr (kBf16)
      return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(rp)[e]) << 16);
    else
      return reinterpret_cast<const float*>(rp)[e];
  };
  // the data-independent Philox words, while the rows are in flight (threads
  // 384..447, warps that hold a row only when there are more than 12):
  // every position's acceptance uniform, every (position, group) exponential
  // of this slice's race groups
  {
    const int t = tid - 384;
    const int g0 = v0 / kRaceGroup, nlg = (n + kRaceGroup - 1) / kRaceGroup;
    if (t >= 0 && t < 64) {
      if (t < g) sm.uacc[t] = static_cast<float>(accept_uniform(sd_block(p, b, kTagAccept, t, t).x));
      for (int u = t; u < (g + 1) * nlg; u += 64)
        sm.gE[u] = exponential_from_bits(sd_block(p, b, kTagGroup, u / nlg, g0 + u % nlg).x);
    }
  }
  float zp = __int_as_float(0x7fc00000), zq = zp;
  if (ti < g && tvalid && !greedy && xi >= 0 && xi < V) {
    zp = logit_at<kBf16>(grow(ti), xi);
    zq = logit_at<kBf16>(grow(g + 1 + ti), xi);
  }
  if (scalar_copies) __syncthreads();  // the scalar head and tail copies

  // ---- 1. row statistics of the slice: a warp per row (q = warp, warp +
  // kSdW, ...; lane l takes entries l, l + 32, ...) as soon as the row has
  // landed: the maximum (NaN-propagating; for greedy rows with its first
  // index), then the scaled sum s = sum_v 2^{(z_v - m) c} against it, each
  // with four independent chains; then one exchange per batch of rows,
  // merged in rank order
  int buf = 0;
  {
    const float c = tvalid && !greedy ? __fdiv_rn(kLog2e, T) : 0.0f;
    for (int q = warp; q < nq; q += kSdW) {
      const bool landed = mbar_wait(&sm.rbar[q], 0);
      const char* rp = srows + static_cast<size_t>(q) * f.rowstride +
                       (reinterpret_cast<uintptr_t>(grow(q) + static_cast<size_t>(v0) * es) & 15u);
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
      if (lane == 0) sm.part[q] = make_float4(m, sum, __int_as_float(arg), __int_as_float(bad));
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    for (int q0 = 0; q0 < nq; q0 += kSdBatch) {
      const int nb = min(kSdBatch, nq - q0);
      exchange_f4(cl, sm, buf, nb, tid < nb ? sm.part[q0 + tid] : make_float4(0.0f, 0.0f, 0.0f, 0.0f));
      if (tid < nb) {
        RowAcc a{-INFINITY, 0.0f, 0x7fffffff, 0};
        for (int r = 0; r < kSdC; ++r) {
          const float4 x = sm.xb[buf][r][tid];
          const RowAcc o{x.x, x.y, __float_as_int(x.z), __float_as_int(x.w)};
          if (greedy) acc_merge<kRowArgmax>(a, o, c); else acc_merge<kRowLse>(a, o, c);
        }
        if (sm.xfail) a.bad = 1;
        sm.rows[q0 + tid] = a;
      }
      exchange_done(sm, buf);
    }
  }

  // ---- 2. the decision, in every CTA (rank 0 writes the outputs)
  if (ti < g) {
    sm.tok[ti] = xi;
    sm.zsel[2 * ti] = zp;
    sm.zsel[2 * ti + 1] = zq;
  }
  __syncthreads();
  if (warp == 0) decide_single<kBf16>(p, b, T, sm.tok, sm.rows, sm.zsel, &sm.si, rank == 0, sm.uacc);
  __syncthreads();
  const SeqInfo si = sm.si;
  const bool draw = (si.mode == kModeResidual && si.j >= 0 && si.j < g) ||
                    (si.mode == kModeBonus && si.j == g);
  if (draw) {  // uniform over the cluster: every CTA took the same decision
    const int j = si.j;
    const float2 nm = make_float2(-si.zmp, -si.zmq), cc = make_float2(si.c, si.c),
                 nl = make_float2(-si.lsp, -si.lsq);
    const char* rt = sm.rowp[j];
    const char* rd = si.mode == kModeResidual ? sm.rowp[g + 1 + j] : rt;
    // weight of local entry e: max(p - q, 0) (resid) or p; 0 past the row
    auto weight = [&](int e, bool resid) -> float {
      if (e >= n) return 0.0f;
      const float2 z = make_float2(zat(rt, e), resid ? zat(rd, e) : -INFINITY);
      const float2 x = __ffma2_rn(__fadd2_rn(z, nm), cc, nl);
      const float pv = ex2_approx(x.x);
      return resid ? fmaxf(pv - ex2_approx(x.y), 0.0f) : pv;
    };
    const int g0 = v0 / kRaceGroup;                       // first race group of the slice
    const int nlg = (n + kRaceGroup - 1) / kRaceGroup;    // race groups in the slice
    // level 1: each group split into wpg parts (wpg warps per group when
    // the slice has fewer groups than warps); a warp sums its part (lane l:
    // entries 4 l + k, then + 128, ...) in order, a butterfly sums the lanes,
    // and the parts of a group are added in order; the CTA's groups race.
    // Level 2 runs at once in the CTA's best group (the cluster's winner is
    // one of the CTAs' best groups), one Philox block per thread of the
    // first kRaceGroup / 4, and the exchange carries the token with the group.
    int wpg = 1;
    while (wpg * 2 * nlg <= kSdW && wpg < 16) wpg *= 2;
    const int span = kRaceGroup / wpg;  // entries per part
    auto levels = [&](bool resid) -> float4 {
      for (int u = warp; u < nlg * wpg; u += kSdW) {
        const int base = (u / wpg) * kRaceGroup + (u % wpg) * span;
        float s = 0.0f;
        for (int e = 4 * lane; e < span; e += 128)
#pragma unroll
          for (int k = 0; k < 4; ++k) s += weight(base + e + k, resid);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) sm.gpart[u] = s;
      }
      __syncthreads();
      float bw = 0.0f, be = 1.0f;
      int bg = INT_MAX;
      if (tid < nlg) {
        float s = 0.0f;
        for (int k = 0; k < wpg; ++k) s += sm.gpart[tid * wpg + k];
        const int gid = g0 + tid;
        const float e = sm.gE[j * nlg + tid];  // drawn in the prologue
        if (race_better(s, e, gid, bw, be, bg)) {
          bw = s;
          be = e;
          bg = gid;
        }
      }
      race_reduce<kSdT>(bw, be, bg, sm.race);
      int y = -1;
      if (bw > 0.0f) {  // uniform: race_reduce returns the winner to every thread
        float ew = 0.0f, ee = 1.0f;
        int ei = INT_MAX;
        if (tid < kRaceGroup / 4) {
          const int blk = bg * (kRaceGroup / 4) + tid;  // global Philox block
          const uint4 rnd = sd_block(p, b, kTagGumbel, j, blk);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float w = weight(4 * blk + k - v0, resid);
            if (!(w > 0.0f)) continue;
            const float e = exponential_from_bits(word_of(rnd, k));
            if (race_better(w, e, 4 * blk + k, ew, ee, ei)) {
              ew = w;
              ee = e;
              ei = 4 * blk + k;
            }
          }
        }
        race_reduce<kSdT>(ew, ee, ei, sm.race);
        y = ei;
      }
      exchange_f4(cl, sm, buf, 1, make_float4(bw, be, __int_as_float(bg), __int_as_float(y)));
      float4 best = make_float4(0.0f, 1.0f, __int_as_float(INT_MAX), __int_as_float(-1));
      for (int r = 0; r < kSdC; ++r) {
        const float4 x = sm.xb[buf][r][0];
        if (race_better(x.x, x.y, __float_as_int(x.z), best.x, best.y, __float_as_int(best.z))) best = x;
      }
      exchange_done(sm, buf);
      return best;
    };
    float4 best = levels(si.mode == kModeResidual);
    if (si.mode == kModeResidual && !(best.x > 0.0f)) best = levels(false);  // the residual vanished: draw from p_j
    if (rank == 0 && tid == 0 && best.x > 0.0f && !sm.xfail)
      p.out_tokens[static_cast<size_t>(b) * (g + 1) + j] = __float_as_int(best.w);
  }
  // every staged row has landed (rows a greedy sequence never read included)
  if (tid == 0)
    for (int q = nq; q < nall; ++q) (void)mbar_wait(&sm.rbar[q], 0);
  cl.sync();  // no CTA leaves while another may still address its shared memory
}

// ------------------------------------------------------------------ launch
namespace {
constexpr size_t kMaxDynSmem = 227 * 1024;

struct SdShape {
  int slice, rowstride;
  size_t smem;
};

SdShape sd_shape(int gamma, int V, int dtype) {
  const size_t es = dtype == SV_BF16 ? 2 : 4;
  const int ng = (V + kRaceGroup - 1) / kRaceGroup;
  SdShape s{};
  s.slice = (ng + kSdC - 1) / kSdC * kRaceGroup;
  s.rowstride = static_cast<int>((static_cast<size_t>(s.slice) * es + 16 + 15) / 16 * 16);
  s.smem = kSdFixed + static_cast<size_t>(2 * gamma + 1) * s.rowstride;
  return s;
}

// Clusters of the kernel (at this shared memory size) that can be resident
// at once on the current device; 0 if none (asked once per device, variant
// and size class).
template <typename Kernel>
int sd_clusters(Kernel kernel, size_t smem) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxDynSmem)) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(kSdC);
  cfg.blockDim = dim3(kSdT);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSdC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return nclusters;
}

// Resident clusters for a shape: the occupancy at its shared-memory size
// rounded up to 8 KB, asked once per device, variant and size.
int sd_capacity(bool bf16, size_t smem) {
  constexpr size_t kStep = 8 * 1024;
  constexpr int kClasses = static_cast<int>((kMaxDynSmem + kStep - 1) / kStep) + 1;
  static std::atomic<int> cap[2][kClasses][64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  const int cls = static_cast<int>((smem + kStep - 1) / kStep);
  if (cls >= kClasses) return 0;
  std::atomic<int>& slot = cap[bf16 ? 1 : 0][cls][dev];
  int v = slot.load(std::memory_order_relaxed);
  if (v == 0) {
    const size_t probe = static_cast<size_t>(cls) * kStep < kMaxDynSmem ? static_cast<size_t>(cls) * kStep : kMaxDynSmem;
    const int n = bf16 ? sd_clusters(sd_cluster_kernel<true>, probe) : sd_clusters(sd_cluster_kernel<false>, probe);
    v = n > 0 ? n : -1;
    slot.store(v, std::memory_order_relaxed);
  }
  return v > 0 ? v : 0;
}
}  // namespace

bool small_path(int B, int gamma, int V, int dtype) {
  const SdShape sh = sd_shape(gamma, V, dtype);
  if (sh.smem > kMaxDynSmem || sh.slice > kSdMaxSlice) return false;
  return B >= 1 && B <= sd_capacity(dtype == SV_BF16, sh.smem);
}

int launch_small(const CallParams& p1, int dtype, cudaStream_t stream) {
  const SdShape sh = sd_shape(p1.gamma, p1.V, dtype);
  SdParams f{};
  f.p = p1;
  f.slice = sh.slice;
  f.rowstride = sh.rowstride;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(p1.B) * kSdC);
  cfg.blockDim = dim3(kSdT);
  cfg.dynamicSmemBytes = sh.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSdC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = dtype == SV_BF16 ? cudaLaunchKernelEx(&cfg, sd_cluster_kernel<true>, f)
                                         : cudaLaunchKernelEx(&cfg, sd_cluster_kernel<false>, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "small-batch cluster kernel launch failed: %s", cudaGetErrorString(e));
  return check_launch("verify (small batch)");
}

}  // namespace sv
