// sv_single.cu -- single-draft verification: a row kernel and a draw
// kernel per call, chained by programmatic dependent launch (small batches of
// narrow rows take the one-cluster-per-sequence kernel of sv_small.cu
// instead; launch_single chooses).
//
// Row kernel (FlashSpec, Methodology s.1): one CTA per (sequence, position,
// vocabulary segment) streams the target row and the draft row of that
// position over the segment with 16-byte loads issued up front (and each
// row's next tile requested into L2 by a bulk prefetch), reduces the
// maximum and the temperature-scaled softmax sum of both rows, picks up the
// draft token's two logits, and publishes one partial.  The CTA that
// completes a sequence (arrival ticket) combines its partials and makes the
// decision: the two log-probabilities of every draft token, the Philox
// acceptance uniforms, the first rejection by warp ballot (FlexDraft,
// Problem definition).
// Draw kernel (Speculative Speculative Decoding, s.2 Saguaro sampling): once
// its sequence's decision is published (a flag the row kernel sets; the draw
// grid may start while the row kernel's last CTAs run), the correction token is
// drawn from max(p_j - q_j, 0), or the bonus token from p_gamma, by a
// two-level exponential race: vocabulary groups of 1024 entries race with
// their summed weights and one Philox exponential each, then the entries of
// the winning group race with per-entry Philox noise.  Several CTAs per
// sequence sum the groups; the CTA that completes a sequence runs the second
// level.
// The row kernel waits on no other CTA (arrival tickets only); a draw CTA
// waits, with a time limit, for one flag that a row-kernel CTA already
// running sets.
// Vocabulary shards (the kShard instantiations): the row kernel runs on one
// shard's columns and its completing CTA exports the shard's merged row
// statistics; after the caller's all-gather, every draw CTA merges all
// shards' records and decides, the race runs over the shard's groups with
// global Philox keys, and the completing CTA exports the shard's candidate;
// after a second all-gather a pick kernel takes the winner.  No wait on
// another CTA in that path.
#include <atomic>
#include <climits>

#include "sv_decide.cuh"
#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"
#include "sv_stream.cuh"

namespace sv {

// ------------------------------------------------------------------ layout
constexpr int kRowThreads = kTileThreads;  // 256
constexpr int kDrawThreads = 256;
constexpr int kDrawWaves = 4;              // about this many waves of draw CTAs per call
constexpr int kPrefetchTiles = 1;          // row tiles requested into L2 ahead of the loads
static_assert(kRowThreads == kDrawThreads, "one thread count for both kernels");

struct SingleParams {
  CallParams p1;       // inputs, outputs, decision state
  RacePartial* part2;   // [B][nc2] draw partials
  unsigned* ticket2;    // [B] draw arrivals
  unsigned* ready;      // [B] decision published (set by the row kernel, cleared by the draw kernel)
  int nc2;              // draw CTAs per sequence
  int gpc;              // race groups per draw CTA
  int nseg;             // row segments per row
  int tiles;            // kTileVec-vector tiles covering a row's body; segment s
                        // covers tiles [s tiles / nseg, (s + 1) tiles / nseg)
  float4* pairpart;     // [B][gamma + 1][nseg] x {target, draft} partials
  float* zx;            // [B][gamma][nseg][2] draft token's target / draft logit
  // vocabulary shards (kShard kernels only): this shard's first column, the
  // full vocabulary, the shard's statistics record and race candidates
  int voff;
  int vfull;
  float4* xstats;       // [B][gamma + 1][3]
  ShardCand* cand;      // [B]
  const float4* allstats;  // [nshards][B][gamma + 1][3]: the gathered records
  int nshards;
};

template <bool kBf16>
__device__ __forceinline__ const char* target_row(const CallParams& p, int b, int i) {
  constexpr size_t es = kBf16 ? 2 : 4;
  return static_cast<const char*>(p.target) +
         (static_cast<size_t>(b) * (p.gamma + 1) + i) * static_cast<size_t>(p.V) * es;
}
template <bool kBf16>
__device__ __forceinline__ const char* draft_row(const CallParams& p, int b, int i) {
  constexpr size_t es = kBf16 ? 2 : 4;
  return static_cast<const char*>(p.draft) +
         (static_cast<size_t>(b) * p.gamma + i) * static_cast<size_t>(p.V) * es;
}

__device__ __forceinline__ void pdl_wait_and_release() {
  // Wait for the previous grid in the stream (programmatic dependent launch),
  // then let the next one start launching its CTAs.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
}

// Empty partials: softmax rows carry R = -inf in the index slot.
__device__ __forceinline__ RowAcc empty_lse_acc() {
  return RowAcc{-INFINITY, 0.0f, __float_as_int(-INFINITY), 0};
}
__device__ __forceinline__ RowAcc empty_argmax_acc() { return RowAcc{-INFINITY, 0.0f, 0x7fffffff, 0}; }

// Block reduction of the two rows' accumulators: a butterfly within each
// warp, then warp 0 merges the 8 warp results of each row by a 3-step
// butterfly (lanes 0-7 row A, lanes 8-15 row B).  One barrier; the result is
// valid in thread 0.
__device__ __forceinline__ void reduce_pair(RowAcc& A, RowAcc& B, bool argmaxA, RowAcc* scratch) {
  constexpr int W = kRowThreads / 32;  // 8 warps
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  warp_merge(A, argmaxA);
  warp_merge(B, false);
  if (lane == 0) {
    scratch[warp] = A;
    scratch[W + warp] = B;
  }
  block_sync<kRowThreads>();
  if (warp == 0) {
    const bool rowB = lane >= W;
    RowAcc v = lane < 2 * W ? scratch[lane] : empty_lse_acc();
    group_merge<W>(v, rowB ? false : argmaxA);
    const RowAcc vb = shfl_xor_acc(v, W);  // lane 0 receives lane 8's row-B result
    if (lane == 0) {
      A = v;
      B = vb;
    }
  }
}

// The softmax sum relative to the row maximum, s = S 2^{R - m c}, from a
// merged softmax partial {m, S, R}.  R - m c lies in [0, 1) up to rounding
// (R is the reference of the row maximum), so one ex2 of that small argument
// (computed in fp64) keeps the relative error near 2^-22.
__device__ __forceinline__ float sum_rel_max(const RowAcc& a, float c) {
  const float R = __int_as_float(a.arg);
  if (!isfinite(a.m) || !isfinite(R)) return a.s;  // invalid row: left to the decision
  const float e = static_cast<float>(static_cast<double>(R) - static_cast<double>(a.m) * static_cast<double>(c));
  return a.s * ex2_approx(e);
}

// Merge, by one warp, the nseg segment partials of position i of sequence b:
// target row A, draft row B (raw {m, S, R} or {m, -, argmax, bad}), and the
// draft token's two logits (NaN where no segment holds the token).
__device__ __forceinline__ void merge_segments(const SingleParams& f, int b, int i, bool argmaxA,
                                               RowAcc& A, RowAcc& B, float& zt, float& zd) {
  const int lane = threadIdx.x & 31;
  const int g = f.p1.gamma;
  A = argmaxA ? empty_argmax_acc() : empty_lse_acc();
  B = empty_lse_acc();
  zt = __int_as_float(0x7fc00000);
  zd = zt;
  const float4* pp = f.pairpart + (static_cast<size_t>(b) * (g + 1) + i) * f.nseg * 2;
  const float* zp = f.zx + (static_cast<size_t>(b) * g + i) * f.nseg * 2;
  for (int q = lane; q < f.nseg; q += 32) {
    const float4 a = __ldcg(pp + 2 * q), d = __ldcg(pp + 2 * q + 1);
    merge_ref(A, RowAcc{a.x, a.y, __float_as_int(a.z), __float_as_int(a.w)}, argmaxA);
    merge_ref(B, RowAcc{d.x, d.y, __float_as_int(d.z), __float_as_int(d.w)}, false);
    if (i < g) {
      // the draft token's logits: the one segment that holds it reports them
      const float za = __ldcg(zp + 2 * q), zb = __ldcg(zp + 2 * q + 1);
      if (za == za) zt = za;
      if (zb == zb) zd = zb;
    }
  }
  warp_merge(A, argmaxA);
  warp_merge(B, false);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float a = __shfl_xor_sync(0xffffffffu, zt, off);
    const float d = __shfl_xor_sync(0xffffffffu, zd, off);
    if (zt != zt) zt = a;
    if (zd != zd) zd = d;
  }
}

// Combine the nseg segment partials of every position of sequence b into the
// row table rows[] (target rows 0..gamma, then draft rows), and pick up the
// draft tokens' logits (zsel[2i], zsel[2i+1]).  argmaxA and c describe the
// sequence (greedy or softmax, c = log2(e) / T).
__device__ __forceinline__ void combine_pairs(const SingleParams& f, int b, bool argmaxA, float c,
                                              RowAcc* rows, float* zsel) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = f.p1.gamma;
  for (int i = warp; i <= g; i += kRowThreads / 32) {
    RowAcc A, B;
    float zt, zd;
    merge_segments(f, b, i, argmaxA, A, B, zt, zd);
    if (lane == 0) {
      if (!argmaxA) A.s = sum_rel_max(A, c);
      B.s = sum_rel_max(B, c);
      rows[i] = A;
      if (i < g) {
        rows[g + 1 + i] = B;
        zsel[2 * i] = zt;
        zsel[2 * i + 1] = zd;
      }
    }
  }
  block_sync<kRowThreads>();
}

// Vocabulary shards: the shard's record of sequence b, per position the
// merged target and draft partials as they merge across shards (raw, argmax
// as a global index) and the draft token's two logits.
__device__ __forceinline__ void export_pairs(const SingleParams& f, int b, bool argmaxA) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = f.p1.gamma;
  for (int i = warp; i <= g; i += kRowThreads / 32) {
    RowAcc A, B;
    float zt, zd;
    merge_segments(f, b, i, argmaxA, A, B, zt, zd);
    if (lane == 0) {
      if (argmaxA && A.arg != 0x7fffffff) A.arg += f.voff;
      float4* o = f.xstats + (static_cast<size_t>(b) * (g + 1) + i) * 3;
      o[0] = make_float4(A.m, A.s, __int_as_float(A.arg), __int_as_float(A.bad));
      o[1] = make_float4(B.m, B.s, __int_as_float(B.arg), __int_as_float(B.bad));
      o[2] = make_float4(zt, zd, 0.0f, 0.0f);
    }
  }
}

// Head (entries before the first 16-byte boundary) and tail (after the last)
// of a row, read as scalars by the first / last segment's CTA.
template <bool kBf16>
__device__ __forceinline__ void row_edges(const char* rp, int V, const RowGeom<kBf16>& g, bool argmax,
                                          float c, bool head, bool tail, int xg, float* zx,
                                          RunAcc& acc) {
  const int tid = threadIdx.x;
  if (head)
    for (int v = tid; v < g.head; v += kRowThreads) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) *zx = z;
      if (argmax) argmax_scalar(acc, z, v); else lse_scalar(acc, z, c);
    }
  if (tail)
    for (int v = g.tail0 + tid; v < V; v += kRowThreads) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) *zx = z;
      if (argmax) argmax_scalar(acc, z, v); else lse_scalar(acc, z, c);
    }
}

// The body vector that holds entry xg of a row, if this thread loads it within
// the segment [k0, k1); -1 otherwise.
template <bool kBf16>
__device__ __forceinline__ int owned_vector(const RowGeom<kBf16>& g, int xg, int k0, int k1) {
  if (xg < g.head || xg >= g.tail0) return -1;
  const int k = (xg - g.head) / Vec16<kBf16>::kN;
  if (k < k0 || k >= k1 || (k - k0) % kRowThreads != static_cast<int>(threadIdx.x)) return -1;
  return k;
}

template <bool kBf16>
__device__ __forceinline__ void pick_logit(const uint4 (&r)[kTileRegs], int own, int kb, int xg,
                                           const RowGeom<kBf16>& g, float* zx) {
  if (own < kb || own >= kb + kTileVec) return;
  const int j = (own - kb) / kRowThreads;
  const int e = (xg - g.head) % Vec16<kBf16>::kN;
#pragma unroll
  for (int q = 0; q < kTileRegs; ++q)  // compile-time q keeps r[] in registers
    if (q == j) *zx = Vec16<kBf16>::at(r[q], e);
}

// --------------------------------------------------------------- row kernel
// Grid: one CTA per (row pair, segment), blockIdx.x = (b (gamma + 1) + i)
// nseg + seg: a sequence's CTAs are consecutive, so sequences complete in
// order of b while the kernel runs.  kShard: the rows are one vocabulary
// shard (columns [voff, voff + V) of vfull), and the CTA that completes a
// sequence writes the shard's record instead of deciding.
template <bool kBf16, bool kShard = false>
__global__ void __launch_bounds__(kRowThreads, 4) rows_kernel(const __grid_constant__ SingleParams f) {
  __shared__ RowAcc rows[kMaxRowsPerSeq];
  __shared__ RowAcc scratch[2 * (kRowThreads / 32)];
  __shared__ float s_zx[2];
  __shared__ float s_zsel[2 * SV_MAX_GAMMA];
  __shared__ int s_tok[SV_MAX_GAMMA];
  __shared__ int s_last;
  pdl_wait_and_release();
  const CallParams& p = f.p1;
  const int tid = threadIdx.x;
  const int pair = static_cast<int>(blockIdx.x) / f.nseg;
  const int seg = static_cast<int>(blockIdx.x) - pair * f.nseg;
  const int b = pair / (p.gamma + 1);
  const int i = pair - b * (p.gamma + 1);
  const float T = __ldg(p.temps + b);
  const int modeA = row_mode(T, true);
  const bool argmaxA = modeA == kRowArgmax;
  const bool loadA = modeA != kRowSkip;
  const bool loadB = i < p.gamma && row_mode(T, false) == kRowLse;
  const float c = modeA == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
  int xg = -1;
  if (modeA == kRowLse && i < p.gamma) {
    const int xt = __ldg(p.tokens + static_cast<size_t>(b) * p.gamma + i);
    if constexpr (kShard) {
      const int xl = xt - f.voff;  // the token's column in this shard
      if (xt >= 0 && xt < f.vfull && xl >= 0 && xl < p.V) xg = xl;
    } else {
      if (xt >= 0 && xt < p.V) xg = xt;
    }
  }
  if (tid == 0) s_zx[0] = s_zx[1] = __int_as_float(0x7fc00000);  // NaN: "not in this segment"
  // the sequence's draft tokens, for the decision if this CTA completes it
  for (int k = tid; k < p.gamma; k += kRowThreads) s_tok[k] = __ldg(p.tokens + static_cast<size_t>(b) * p.gamma + k);
  block_sync<kRowThreads>();

  RunAcc accA, accB;
  accA.reset();
  accB.reset();
  const char* rpA = target_row<kBf16>(p, b, i);
  const char* rpB = loadB ? draft_row<kBf16>(p, b, i) : rpA;
  const RowGeom<kBf16> gA(rpA, p.V), gB(rpB, p.V);
  const int k0 = static_cast<int>(static_cast<long long>(seg) * f.tiles / f.nseg) * kTileVec;
  const int kseg1 = static_cast<int>(static_cast<long long>(seg + 1) * f.tiles / f.nseg) * kTileVec;
  const int a1 = min(gA.nvec, kseg1), b1 = min(gB.nvec, kseg1);
  const uint4* vA = gA.body(rpA);
  const uint4* vB = gB.body(rpB);
  const int ownA = owned_vector<kBf16>(gA, xg, k0, a1);
  const int ownB = owned_vector<kBf16>(gB, xg, k0, b1);
  const int kend = max(loadA ? a1 : k0, loadB ? b1 : k0);
  // L2 prefetch kPrefetchTiles tiles ahead of the loads (one bulk request
  // per row and tile, issued by lane 0 of warps 0 and 1), so DRAM keeps
  // streaming while the registers wait on the current tile.
  auto prefetch = [&](int kp) {
    if (tid == 0 && loadA && kp < a1) prefetch_l2(vA + kp, static_cast<uint32_t>(min(kTileVec, a1 - kp)) * 16u);
    if (tid == 32 && loadB && kp < b1) prefetch_l2(vB + kp, static_cast<uint32_t>(min(kTileVec, b1 - kp)) * 16u);
  };
#pragma unroll
  for (int d = 1; d < kPrefetchTiles; ++d) prefetch(k0 + d * kTileVec);
  for (int kb = k0; kb < kend; kb += kTileVec) {
    if (kPrefetchTiles > 0) prefetch(kb + kPrefetchTiles * kTileVec);
    uint4 ra[kTileRegs], rb[kTileRegs];
    if (loadA) load_tile<kBf16>(vA, kb, a1, ra);
    if (loadB) load_tile<kBf16>(vB, kb, b1, rb);
    if (loadA) {
      pick_logit<kBf16>(ra, ownA, kb, xg, gA, &s_zx[0]);
      if (argmaxA)
        argmax_tile<kBf16>(accA, ra, gA.head + (kb + tid) * Vec16<kBf16>::kN);
      else
        lse_tile<kBf16>(accA, ra, c);
    }
    if (loadB) {
      pick_logit<kBf16>(rb, ownB, kb, xg, gB, &s_zx[1]);
      lse_tile<kBf16>(accB, rb, c);
    }
  }
  const bool first = seg == 0, last = seg == f.nseg - 1;
  if (loadA && (first || last))
    row_edges<kBf16>(rpA, p.V, gA, argmaxA, c, first, last, xg, &s_zx[0], accA);
  if (loadB && (first || last))
    row_edges<kBf16>(rpB, p.V, gB, false, c, first, last, xg, &s_zx[1], accB);

  RowAcc A = argmaxA ? accA.argmax_row() : accA.lse_row(), B = accB.lse_row();
  reduce_pair(A, B, argmaxA, scratch);
  if (tid == 0) {
    float4* pp = f.pairpart + ((static_cast<size_t>(b) * (p.gamma + 1) + i) * f.nseg + seg) * 2;
    pp[0] = make_float4(A.m, A.s, __int_as_float(A.arg), __int_as_float(A.bad));
    pp[1] = make_float4(B.m, B.s, __int_as_float(B.arg), __int_as_float(B.bad));
    if (i < p.gamma) {
      float* z = f.zx + ((static_cast<size_t>(b) * p.gamma + i) * f.nseg + seg) * 2;
      z[0] = s_zx[0];
      z[1] = s_zx[1];
    }
    // release this CTA's partial; the last arriver also acquires the others'
    const unsigned tk = ticket_acq_rel(p.ticket + b);
    const unsigned arrivals = static_cast<unsigned>((p.gamma + 1) * f.nseg);
    s_last = (tk == arrivals - 1);
    if (s_last) p.ticket[b] = 0;  // leave the counter at zero for the next call
  }
  block_sync<kRowThreads>();  // orders the other threads after thread 0's acquire
  if (!s_last) return;
  if constexpr (kShard) {
    export_pairs(f, b, argmaxA);
    return;
  }
  combine_pairs(f, b, argmaxA, c, rows, s_zsel);
  if (tid < 32) {
    decide_single<kBf16>(p, b, T, s_tok, rows, s_zsel, p.info + b, true, nullptr);
    // publish the decision: every lane's writes, then the flag (release)
    __threadfence();
    __syncwarp();
    if (tid == 0) st_release(f.ready + b, 1u);
  }
}

// -------------------------------------------------------------- draw kernel
// The 4 logits of Philox block g of a row, kept packed until used; entries
// at or beyond V read as -inf.
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
  __device__ __forceinline__ void load_vec(const char* row, int g) {
    r = __ldg(reinterpret_cast<const uint2*>(row) + g);
  }
  __device__ __forceinline__ float at(int w) const {
    const uint32_t x = w < 2 ? r.x : r.y;
    return (w & 1) ? bf16_hi(x) : bf16_lo(x);
  }
  __device__ __forceinline__ void set_neg_inf() { r = make_uint2(0xFF80FF80u, 0xFF80FF80u); }
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
  __device__ __forceinline__ void load_vec(const char* row, int g) {
    r = __ldg(reinterpret_cast<const float4*>(row) + g);
  }
  __device__ __forceinline__ float at(int w) const {
    return w == 0 ? r.x : (w == 1 ? r.y : (w == 2 ? r.z : r.w));
  }
  __device__ __forceinline__ void set_neg_inf() { r = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY); }
};

// Philox stream of one draw: blocks (c0 = g) of the keyed counter
// (g, b, step, tag << 24 | j) under key (lo32 seed, hi32 seed).
struct RaceKey {
  uint32_t k0, k1, b, step, c3;
  __device__ __forceinline__ uint4 block(int g) const {
    return philox4x32_10(make_uint4(static_cast<uint32_t>(g), b, step, c3), k0, k1);
  }
};

// Sequence b's draw: the row(s) it reads and the constants of its weights
// w_v = max(p_v - q_v, 0) (residual) or p_v (bonus), with
// p_v = 2^{(z_v - zmp) c - lsp} and q_v = 2^{(y_v - zmq) c - lsq}.
template <bool kBf16>
struct DrawRow {
  const char* trow;
  const char* drow;
  bool tvec, dvec, resid;
  int V, nblocks;
  float2 nm, cc, nl;
  __device__ __forceinline__ DrawRow(const CallParams& p, const SeqInfo& si, int b, bool resid_) {
    constexpr uintptr_t kVecAlign = kBf16 ? 8 : 16;
    resid = resid_;
    trow = target_row<kBf16>(p, b, si.j);
    drow = resid ? draft_row<kBf16>(p, b, si.j) : trow;
    tvec = (reinterpret_cast<uintptr_t>(trow) % kVecAlign) == 0;
    dvec = (reinterpret_cast<uintptr_t>(drow) % kVecAlign) == 0;
    V = p.V;
    nblocks = (p.V + 3) / 4;
    nm = make_float2(-si.zmp, -si.zmq);
    cc = make_float2(si.c, si.c);
    nl = make_float2(-si.lsp, -si.lsq);
  }
  // Logits of Philox block g (entries 4g .. 4g + 3; -inf past the row).
  __device__ __forceinline__ void load(int g, Block4<kBf16>& tb, Block4<kBf16>& db) const {
    tb.set_neg_inf();
    db.set_neg_inf();
    if (g < nblocks) {
      tb.load(trow, tvec, V, g);
      if (resid) db.load(drow, dvec, V, g);
    }
  }
  // The same for a block known to lie inside the row, rows vector-aligned.
  __device__ __forceinline__ void load_fast(int g, Block4<kBf16>& tb, Block4<kBf16>& db) const {
    tb.load_vec(trow, g);
    if (resid) db.load_vec(drow, g); else db.set_neg_inf();
  }
  // Group gid lies inside the row and both rows take vector loads.
  __device__ __forceinline__ bool fast(int gid) const {
    return tvec && (dvec || !resid) && (gid + 1) * kRaceGroup <= V;
  }
  // The four weights: the target and draft value of an entry travel as one
  // packed pair through the shift and the scale.
  __device__ __forceinline__ float4 weights(const Block4<kBf16>& tb, const Block4<kBf16>& db) const {
    float w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 e = __ffma2_rn(__fadd2_rn(make_float2(tb.at(k), db.at(k)), nm), cc, nl);
      w[k] = ex2_approx(e.x);
      if (resid) w[k] = fmaxf(w[k] - ex2_approx(e.y), 0.0f);
    }
    return make_float4(w[0], w[1], w[2], w[3]);
  }
};

// Level 1 of the draw, by one warp: the groups gid = g0, g0 + gstride, ...
// below g1.  A group's 1024 entries are 8 passes of 32 lanes x 4 entries
// (lane l of pass t holds Philox block 256 gid + 32 t + l), loaded 8 (bf16) or
// 4 (fp32) passes at a time before any is used; each lane sums its 32 weights in order, then a butterfly over
// the lanes gives every lane the same W_g.  The k-th group's W_g stays with
// lane k % 32; every 32 groups (and at the end) those lanes draw their
// groups' exponentials in parallel and enter the race.  Returns the warp's
// winner in (bw, be, bi) (bi: the group index).  goff: the global index of
// the row's group 0 (a vocabulary shard's offset / 1024; 0 for whole rows):
// the race keys and bi are global, the loads local.
template <bool kBf16>
__device__ __forceinline__ void race_groups(const DrawRow<kBf16>& r, const RaceKey& gkey, int g0,
                                            int gstride, int g1, float& bw, float& be, int& bi,
                                            int goff) {
  constexpr int kPasses = kRaceGroup / 128;
  constexpr int kBatch = kBf16 ? 8 : 4;  // passes loaded together (32 registers of logits)
  const int lane = threadIdx.x & 31;
  float myW = 0.0f;
  int myG = -1;
  int k = 0;
  auto enter = [&]() {
    if (myG >= 0) {
      const float e = exponential_from_bits(gkey.block(myG).x);
      if (race_better(myW, e, myG, bw, be, bi)) {
        bw = myW;
        be = e;
        bi = myG;
      }
    }
    myG = -1;
  };
  for (int gid = g0; gid < g1; gid += gstride, ++k) {
    float s = 0.0f;
#pragma unroll
    for (int t0 = 0; t0 < kPasses; t0 += kBatch) {
      Block4<kBf16> tb[kBatch], db[kBatch];
      if (r.fast(gid)) {  // uniform over the warp
#pragma unroll
        for (int t = 0; t < kBatch; ++t) r.load_fast(gid * (kRaceGroup / 4) + (t0 + t) * 32 + lane, tb[t], db[t]);
      } else {
#pragma unroll
        for (int t = 0; t < kBatch; ++t) r.load(gid * (kRaceGroup / 4) + (t0 + t) * 32 + lane, tb[t], db[t]);
      }
#pragma unroll
      for (int t = 0; t < kBatch; ++t) {
        const float4 w = r.weights(tb[t], db[t]);
        s = (((s + w.x) + w.y) + w.z) + w.w;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == (k & 31)) {
      myW = s;
      myG = gid + goff;
    }
    if ((k & 31) == 31) enter();
  }
  enter();
}

// Level 2, by the whole CTA: the entries of global group gid, one Philox
// block per thread (block 256 gid + t), in the race of w_v / E_v with the
// per-entry noise; the row's group 0 is global group goff.  Returns the CTA's
// winner (a global vocabulary index) in every thread.
template <bool kBf16>
__device__ __forceinline__ int race_entries(const DrawRow<kBf16>& r, const RaceKey& ekey, int gid,
                                            float4* scratch, int goff) {
  static_assert(kDrawThreads * 4 == kRaceGroup, "one Philox block per thread");
  const int g = gid * (kRaceGroup / 4) + static_cast<int>(threadIdx.x);  // global block
  Block4<kBf16> tb, db;
  r.load(g - goff * (kRaceGroup / 4), tb, db);
  const float4 w4 = r.weights(tb, db);
  const float w[4] = {w4.x, w4.y, w4.z, w4.w};
  const uint4 rnd = ekey.block(g);
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (!(w[k] > 0.0f)) continue;
    const float e = exponential_from_bits(word_of(rnd, k));
    if (race_better(w[k], e, 4 * g + k, bw, be, bi)) {
      bw = w[k];
      be = e;
      bi = 4 * g + k;
    }
  }
  race_reduce<kDrawThreads>(bw, be, bi, scratch);
  return bi;
}

// Both levels over the whole target row j in one CTA: the draw from p_j
// when the residual max(p_j - q_j, 0) vanished (p_j == q_j to rounding).
// The level-1 winner goes to *win ({w, E, global group}) when win is not
// NULL; -1 when no entry of the row has weight (a vocabulary shard far
// below the row's maximum).
template <bool kBf16>
__device__ __noinline__ int draw_from_target(const CallParams& p, const SeqInfo& si, int b,
                                             const RaceKey& gkey, const RaceKey& ekey, float4* scratch,
                                             int goff, float4* win) {
  const DrawRow<kBf16> prow(p, si, b, false);
  const int ng = (p.V + kRaceGroup - 1) / kRaceGroup;
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
  race_groups<kBf16>(prow, gkey, static_cast<int>(threadIdx.x >> 5), kDrawThreads / 32, ng, bw, be, bi,
                     goff);
  race_reduce<kDrawThreads>(bw, be, bi, scratch);
  if (win) *win = make_float4(bw, be, __int_as_float(bi), 0.0f);
  if (!(bw > 0.0f)) return -1;  // uniform: race_reduce returns the winner to every thread
  return race_entries<kBf16>(prow, ekey, bi, scratch, goff);
}

// Draw kernel.  Grid: nc2 CTAs per sequence; CTA c of sequence b runs level
// 1 over groups [c gpc, (c + 1) gpc) (warp w: groups c gpc + w, + 8, ...),
// publishes its winning group, and the CTA that completes the sequence
// (arrival ticket) combines the nc2 winners and runs level 2 in the winning
// group.  If every residual weight is zero (p_j == q_j to rounding), that CTA
// draws from p_j instead, both levels over the whole row.
// Bounded wait (kWaitLimitNs) for sequence b's decision flag, by one thread.
__device__ __forceinline__ bool wait_ready(const unsigned* flag) {
  if (ld_acquire(flag) != 0u) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    __nanosleep(256);
    if (ld_acquire(flag) != 0u) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ------------------------------------------------- vocabulary shards: decide
// Merge the gathered shards' records of sequence b into the row table rows[]
// (target rows 0..gamma, then draft rows) and the draft tokens' logits
// zsel[]: a warp per position, lane r merging rank r's record, then a
// butterfly -- the same order on every rank, so every rank reaches the same
// bits.  All kDrawThreads threads; ends with a barrier.
__device__ __forceinline__ void merge_shards(const SingleParams& f, int b, bool argmaxA, float c,
                                             RowAcc* rows, float* zsel) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = f.p1.gamma;
  const size_t per_rank = static_cast<size_t>(f.p1.B) * (g + 1) * 3;  // float4s in one record
  for (int i = warp; i <= g; i += kDrawThreads / 32) {
    RowAcc A = argmaxA ? empty_argmax_acc() : empty_lse_acc(), Bq = empty_lse_acc();
    float zt = __int_as_float(0x7fc00000), zd = zt;
    for (int r = lane; r < f.nshards; r += 32) {
      const float4* o = f.allstats + r * per_rank + (static_cast<size_t>(b) * (g + 1) + i) * 3;
      const float4 a = __ldcg(o), d = __ldcg(o + 1), z = __ldcg(o + 2);
      merge_ref(A, RowAcc{a.x, a.y, __float_as_int(a.z), __float_as_int(a.w)}, argmaxA);
      merge_ref(Bq, RowAcc{d.x, d.y, __float_as_int(d.z), __float_as_int(d.w)}, false);
      if (z.x == z.x) zt = z.x;  // the one shard that holds the draft token reports its logits
      if (z.y == z.y) zd = z.y;
    }
    warp_merge(A, argmaxA);
    warp_merge(Bq, false);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float a = __shfl_xor_sync(0xffffffffu, zt, off);
      const float d = __shfl_xor_sync(0xffffffffu, zd, off);
      if (zt != zt) zt = a;
      if (zd != zd) zd = d;
    }
    if (lane == 0) {
      if (!argmaxA) A.s = sum_rel_max(A, c);
      Bq.s = sum_rel_max(Bq, c);
      rows[i] = A;
      if (i < g) {
        rows[g + 1 + i] = Bq;
        zsel[2 * i] = zt;
        zsel[2 * i + 1] = zd;
      }
    }
  }
  block_sync<kDrawThreads>();
}

// kShard: the rows are one vocabulary shard; every CTA first takes its
// sequence's decision from the gathered shards' records, the race runs over
// the shard's groups with global group and entry indices, and the completing
// CTA writes the shard's candidate (its best group with that group's level-2
// winner, or, where the shard's residual has no weight, the same for the race
// over p_j) instead of the token.
template <bool kBf16, bool kShard = false>
__global__ void __launch_bounds__(kDrawThreads, 4) draw_kernel(const __grid_constant__ SingleParams f) {
  __shared__ float4 scratch[kDrawThreads / 32];
  __shared__ int s_last, s_ready;
  // Whole rows: no griddepcontrol.wait -- this grid may start while the row
  // kernel's last CTAs still run, and each CTA waits for its own sequence's
  // decision flag instead.  (It starts only once every row-kernel CTA has
  // started, so the row kernel never waits for SM room held by this grid.)
  const int b = blockIdx.x / f.nc2;
  const int chunk = blockIdx.x - b * f.nc2;
  const int warp = threadIdx.x >> 5;
  const CallParams& p = f.p1;
  SeqInfo si{};
  si.mode = kModeNone;
  if constexpr (kShard) {
    // Vocabulary shards: every CTA of the sequence takes the decision from
    // the gathered records (no wait on another CTA); chunk 0 writes the
    // outputs.  The records may come from the previous grid in the stream.
    __shared__ RowAcc rows[kMaxRowsPerSeq];
    __shared__ float s_zsel[2 * SV_MAX_GAMMA];
    __shared__ int s_tok[SV_MAX_GAMMA];
    __shared__ CallParams s_p;
    __shared__ SeqInfo s_si;
    pdl_wait_and_release();
    const float T = __ldg(p.temps + b);
    const int modeA = row_mode(T, true);
    const float c = modeA == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
    for (int k = threadIdx.x; k < p.gamma; k += kDrawThreads)
      s_tok[k] = __ldg(p.tokens + static_cast<size_t>(b) * p.gamma + k);
    if (threadIdx.x == 0) {
      s_p = p;
      s_p.V = f.vfull;  // draft tokens are checked against the full vocabulary
    }
    merge_shards(f, b, modeA == kRowArgmax, c, rows, s_zsel);
    if (warp == 0) decide_single<kBf16>(s_p, b, T, s_tok, rows, s_zsel, &s_si, chunk == 0, nullptr);
    block_sync<kDrawThreads>();
    si = s_si;
  } else {
    asm volatile("griddepcontrol.launch_dependents;");
    if (threadIdx.x == 0) s_ready = wait_ready(f.ready + b) ? 1 : 0;
    block_sync<kDrawThreads>();  // orders the other threads after thread 0's acquire
  }
  if (!kShard && s_ready) {
    const float4* ip = reinterpret_cast<const float4*>(p.info + b);
    const float4 w0 = __ldcg(ip), w1 = __ldcg(ip + 1);
    si.mode = __float_as_int(w0.x);
    si.j = __float_as_int(w0.y);
    si.zmp = w0.z;
    si.zmq = w0.w;
    si.c = w1.x;
    si.lsp = w1.y;
    si.lsq = w1.z;
  } else if (!kShard && chunk == 0) {
    // the decision never came (a wait ran out of time): no result
    for (int i = threadIdx.x; i <= p.gamma; i += kDrawThreads)
      p.out_tokens[static_cast<size_t>(b) * (p.gamma + 1) + i] = -1;
    if (threadIdx.x == 0) p.accept_len[b] = -1;
  }
  const bool draw = (si.mode == kModeResidual && si.j >= 0 && si.j < p.gamma) ||
                    (si.mode == kModeBonus && si.j == p.gamma);
  const uint32_t k0 = static_cast<uint32_t>(p.seed), k1 = static_cast<uint32_t>(p.seed >> 32);
  const RaceKey gkey{k0, k1, static_cast<uint32_t>(b), p.step, (kTagGroup << 24) | static_cast<uint32_t>(si.j)};
  const RaceKey ekey{k0, k1, static_cast<uint32_t>(b), p.step, (kTagGumbel << 24) | static_cast<uint32_t>(si.j)};
  const int ng = (p.V + kRaceGroup - 1) / kRaceGroup;
  const int goff = kShard ? f.voff / kRaceGroup : 0;
  float bw = 0.0f, be = 1.0f;
  int bi = INT_MAX;
  if (draw) {  // uniform
    const DrawRow<kBf16> row(p, si, b, si.mode == kModeResidual);
    const int gc0 = chunk * f.gpc;
    race_groups<kBf16>(row, gkey, gc0 + warp, kDrawThreads / 32, min(ng, gc0 + f.gpc), bw, be, bi,
                       goff);
    race_reduce<kDrawThreads>(bw, be, bi, scratch);
  }
  // Every CTA of the sequence arrives (drawing or not), so the last one can
  // clear the flag and the counter for the next call.
  if (threadIdx.x == 0) {
    RacePartial* pp = f.part2 + static_cast<size_t>(b) * f.nc2 + chunk;
    if (draw) *reinterpret_cast<float4*>(pp) = make_float4(bw, be, __int_as_float(bi), 0.0f);
    const unsigned t = ticket_acq_rel(f.ticket2 + b);
    s_last = (t == static_cast<unsigned>(f.nc2 - 1));
    if (s_last) {
      f.ticket2[b] = 0;
      f.ready[b] = 0;  // every CTA of the sequence is past its wait
    }
  }
  block_sync<kDrawThreads>();  // orders the other threads after thread 0's acquire
  if (!s_last) return;
  if constexpr (!kShard) {
    if (!draw) return;
  } else if (!draw) {
    if (threadIdx.x == 0) f.cand[b] = ShardCand{0.0f, 1.0f, INT_MAX, -1, kShardNoDraw, si.j, 0, 0};
    return;
  }
  bw = 0.0f;
  be = 1.0f;
  bi = INT_MAX;
  for (int q = threadIdx.x; q < f.nc2; q += kDrawThreads) {
    const float4 g = __ldcg(reinterpret_cast<const float4*>(f.part2 + static_cast<size_t>(b) * f.nc2 + q));
    if (race_better(g.x, g.y, __float_as_int(g.z), bw, be, bi)) {
      bw = g.x;
      be = g.y;
      bi = __float_as_int(g.z);
    }
  }
  race_reduce<kDrawThreads>(bw, be, bi, scratch);
  if constexpr (kShard) {
    ShardCand cd{bw, be, bi, -1, kShardDrawLaw, si.j, 0, 0};
    if (bw > 0.0f) {  // uniform
      const DrawRow<kBf16> row(p, si, b, si.mode == kModeResidual);
      cd.token = race_entries<kBf16>(row, ekey, bi, scratch, goff);
    } else if (si.mode == kModeResidual) {
      // no residual weight in this shard: its candidate of the race over p_j,
      // used only if no shard has residual weight
      float4 w;
      cd.token = draw_from_target<kBf16>(p, si, b, gkey, ekey, scratch, goff, &w);
      cd = ShardCand{w.x, w.y, __float_as_int(w.z), cd.token, kShardTargetRace, si.j, 0, 0};
    }
    if (threadIdx.x == 0) f.cand[b] = cd;
  } else {
    int y;
    if (bw > 0.0f) {  // uniform: race_reduce returns the winner to every thread
      const DrawRow<kBf16> row(p, si, b, si.mode == kModeResidual);
      y = race_entries<kBf16>(row, ekey, bi, scratch, 0);
    } else {
      y = draw_from_target<kBf16>(p, si, b, gkey, ekey, scratch, 0, nullptr);  // the residual vanished
    }
    if (threadIdx.x == 0) p.out_tokens[static_cast<size_t>(b) * (p.gamma + 1) + si.j] = y;
  }
}

// --------------------------------------------------- vocabulary shards: pick
constexpr int kPickThreads = 256;

// The better of two candidates of one kind (exponential race: larger w / E,
// lower group on ties), the token travelling with its group.
__device__ __forceinline__ void pick_better(float& bw, float& be, int& bg, int& bt, float w, float e,
                                            int grp, int t) {
  if (race_better(w, e, grp, bw, be, bg)) {
    bw = w;
    be = e;
    bg = grp;
    bt = t;
  }
}

// One warp per sequence, lane r reading rank r's candidate (and r + 32, ...):
// the winning candidate over the gathered shards' candidates (the draw law's
// when any shard has weight in it, else the race over p_j), written at the
// draw position.  Shards that disagree on the draw (ranks given different
// sequence inputs, or records gathered in different orders) mark the
// sequence invalid.
__global__ void __launch_bounds__(kPickThreads) shard_pick_kernel(const ShardCand* all, int nshards, int B,
                                                                   int gamma, int32_t* accept_len,
                                                                   int32_t* out_tokens) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int b = static_cast<int>(blockIdx.x) * (kPickThreads / 32) + static_cast<int>(threadIdx.x >> 5);
  if (b >= B) return;  // uniform over the warp
  const ShardCand c0 = all[b];
  float bw[2] = {0.0f, 0.0f}, be[2] = {1.0f, 1.0f};
  int bg[2] = {INT_MAX, INT_MAX}, bt[2] = {-1, -1};
  bool agree = true;
  for (int r = lane; r < nshards; r += 32) {
    const ShardCand c = all[static_cast<size_t>(r) * B + b];
    agree = agree && (c.kind == kShardNoDraw) == (c0.kind == kShardNoDraw) && c.j == c0.j;
    if (c.kind == kShardNoDraw) continue;
    const int k = c.kind == kShardTargetRace ? 1 : 0;
    pick_better(bw[k], be[k], bg[k], bt[k], c.w, c.e, c.group, c.token);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float w = __shfl_xor_sync(0xffffffffu, bw[k], off);
      const float e = __shfl_xor_sync(0xffffffffu, be[k], off);
      const int grp = __shfl_xor_sync(0xffffffffu, bg[k], off);
      const int t = __shfl_xor_sync(0xffffffffu, bt[k], off);
      pick_better(bw[k], be[k], bg[k], bt[k], w, e, grp, t);
    }
  }
  agree = __all_sync(0xffffffffu, agree);
  int32_t* tok = out_tokens + static_cast<size_t>(b) * (gamma + 1);
  if (!agree) {
    for (int i = lane; i <= gamma; i += 32) tok[i] = -1;
    if (lane == 0) accept_len[b] = -1;
    return;
  }
  if (lane != 0 || c0.kind == kShardNoDraw || c0.j < 0 || c0.j > gamma) return;
  tok[c0.j] = bw[0] > 0.0f ? bt[0] : bt[1];
}

// ------------------------------------------------------------------ launch
namespace {
int body_tiles(int V, int dtype) {  // tiles of kTileVec vectors covering a row's body
  const long long vecs = static_cast<long long>(V) * (dtype == SV_BF16 ? 2 : 4) / 16;
  const long long t = (vecs + kTileVec - 1) / kTileVec;
  return t < 1 ? 1 : static_cast<int>(t);
}
}  // namespace

int row_segments(int V, int dtype) { return body_tiles(V, dtype); }  // bound on segments per row

int draw_chunks(int V) {  // upper bound on draw CTAs per sequence: one group per warp
  const int ng = (V + kRaceGroup - 1) / kRaceGroup;
  return (ng + kDrawThreads / 32 - 1) / (kDrawThreads / 32);
}

namespace {
// A host query whose answer is fixed per device (SM count, occupancy), asked
// once per device and kept.  The slots are atomics: threads that call at the
// same time may both ask, and store the same value.
template <typename Query>
int per_device(std::atomic<int> (&slots)[64], int fallback, Query query) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fallback;
  int v = slots[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    v = query(dev);
    if (v <= 0) v = fallback;
    slots[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

int sm_count() {
  static std::atomic<int> slots[64];
  return per_device(slots, 148, [](int dev) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    return n;
  });
}

template <typename Kernel>
int occupancy(Kernel kernel, int threads) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

// Resident row-kernel CTAs per SM.
int row_ctas_per_sm(bool bf16) {
  static std::atomic<int> slots[2][64];
  return bf16 ? per_device(slots[1], 4, [](int) { return occupancy(rows_kernel<true>, kRowThreads); })
              : per_device(slots[0], 4, [](int) { return occupancy(rows_kernel<false>, kRowThreads); });
}

// Resident draw-kernel CTAs per SM.
int draw_ctas_per_sm(bool bf16) {
  static std::atomic<int> slots[2][64];
  return bf16 ? per_device(slots[1], 4, [](int) { return occupancy(draw_kernel<true>, kDrawThreads); })
              : per_device(slots[0], 4, [](int) { return occupancy(draw_kernel<false>, kDrawThreads); });
}

template <typename K, typename P>
cudaError_t launch_pdl(K kernel, dim3 grid, unsigned block, cudaStream_t stream, const P& f) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, f);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;  // retry as an ordinary stream-ordered launch
    e = cudaLaunchKernelEx(&cfg, kernel, f);
  }
  return e;
}

// Row segments: whole tiles, about kRowWaves waves of CTAs over the GPU but
// at most kMaxSegTiles tiles per CTA; balanced so segments differ by at most
// one tile.  Long segments spread each CTA's fixed cost (launch, block
// reduce, ticket) over more streaming; about two waves of four CTAs per SM
// (64 registers a thread) measured best (C2 76.2 us against 83.3 at four
// waves and 77.4 at three).  Draw CTAs: race groups per warp chosen so that the B
// sequences' groups fill about kDrawWaves waves of CTAs (at least one group
// per warp, so a small batch still spreads each row over several CTAs); a
// CTA covers 8 warps' groups.  V is the width of the rows the kernels read.
void set_policy(SingleParams& f, int B, int gamma, int V, int dtype, char* ws, const Layout& lay) {
  const bool bf16 = dtype == SV_BF16;
  {
    constexpr int kRowWaves = 2, kMaxSegTiles = 10;
    const int tiles = body_tiles(V, dtype);
    const long long pairs = static_cast<long long>(B) * (gamma + 1);
    const long long slots = static_cast<long long>(sm_count()) * row_ctas_per_sm(bf16);
    long long st = pairs * tiles / (kRowWaves * slots);
    st = st < 1 ? 1 : (st > kMaxSegTiles ? kMaxSegTiles : st);
    int nseg = static_cast<int>((tiles + st - 1) / st);
    if (nseg > lay.nc) nseg = lay.nc;
    f.nseg = nseg;
    f.tiles = tiles;
  }
  f.pairpart = reinterpret_cast<float4*>(ws + lay.part1);
  f.zx = reinterpret_cast<float*>(ws + lay.resid);
  f.part2 = reinterpret_cast<RacePartial*>(ws + lay.part2);
  f.ticket2 = reinterpret_cast<unsigned*>(ws + lay.ticket2);
  f.ready = reinterpret_cast<unsigned*>(ws + lay.ready);
  {
    const long long ng = (V + kRaceGroup - 1) / kRaceGroup;
    const long long warps = static_cast<long long>(sm_count()) * draw_ctas_per_sm(bf16) * (kDrawThreads / 32);
    long long gpw = (static_cast<long long>(B) * ng + warps * kDrawWaves - 1) / (warps * kDrawWaves);
    if (gpw < 1) gpw = 1;
    const long long gpc = gpw * (kDrawThreads / 32);
    f.gpc = static_cast<int>(gpc < ng ? gpc : ng);
    f.nc2 = static_cast<int>((ng + f.gpc - 1) / f.gpc);  // <= lay.nc2: gpc >= 8 or nc2 == 1
  }
}

// The call's inputs, outputs and the workspace's counters; V is the width of
// the rows (a shard's width for the vocabulary-sharded kernels).
void set_call(CallParams& p1, const void* target, const void* draft, const int32_t* tokens,
              const float* temps, int B, int gamma, int V, uint64_t seed, uint64_t step,
              int32_t* out_accept_len, int32_t* out_tokens, float* out_lp, float* out_lq,
              char* ws, const Layout& lay) {
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
  p1.accept_len = out_accept_len;
  p1.out_tokens = out_tokens;
  p1.out_lp = out_lp;
  p1.out_lq = out_lq;
}
}  // namespace

int launch_single(const void* target, const void* draft, const int32_t* tokens,
                  const float* temps, int B, int gamma, int V, int dtype, uint64_t seed,
                  uint64_t step, int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                  float* out_lq, void* workspace, const Layout& lay, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  SingleParams f{};
  CallParams& p1 = f.p1;
  set_call(p1, target, draft, tokens, temps, B, gamma, V, seed, step, out_accept_len, out_tokens,
           out_lp, out_lq, ws, lay);
  // a batch whose sequences fit one cluster each, in one wave, with every
  // row slice in shared memory: the latency-bound case, one cluster kernel
  if (small_path(B, gamma, V, dtype)) return launch_small(p1, dtype, stream);
  const bool bf16 = dtype == SV_BF16;
  set_policy(f, B, gamma, V, dtype, ws, lay);
  if (static_cast<long long>(B) * f.nc2 > INT_MAX)
    return set_error(SV_ERR_INVALID_ARG, "B x V too large for one launch (draw grid %lld CTAs)",
                     static_cast<long long>(B) * f.nc2);
  const long long ctas1 = static_cast<long long>(B) * (gamma + 1) * f.nseg;
  if (ctas1 > INT_MAX)
    return set_error(SV_ERR_INVALID_ARG, "B x V too large for one launch (row grid %lld CTAs)", ctas1);
  const dim3 grid1(static_cast<unsigned>(ctas1));
  cudaError_t e = bf16 ? launch_pdl(rows_kernel<true>, grid1, kRowThreads, stream, f)
                       : launch_pdl(rows_kernel<false>, grid1, kRowThreads, stream, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "row kernel launch failed: %s", cudaGetErrorString(e));
  const dim3 grid2(static_cast<unsigned>(static_cast<long long>(B) * f.nc2));
  e = bf16 ? launch_pdl(draw_kernel<true>, grid2, kDrawThreads, stream, f)
           : launch_pdl(draw_kernel<false>, grid2, kDrawThreads, stream, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "draw kernel launch failed: %s", cudaGetErrorString(e));
  return check_launch("verify");
}

// ---------------------------------------------------- vocabulary shards: launch
namespace {
int shard_params(SingleParams& f, const void* target, const void* draft, const int32_t* tokens,
                 const float* temps, int B, int gamma, int V, int v0, int Vs, int dtype,
                 uint64_t seed, uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                 float* out_lp, float* out_lq, void* workspace, const Layout& lay) {
  char* ws = static_cast<char*>(workspace);
  set_call(f.p1, target, draft, tokens, temps, B, gamma, Vs, seed, step, out_accept_len, out_tokens,
           out_lp, out_lq, ws, lay);
  set_policy(f, B, gamma, Vs, dtype, ws, lay);
  // a shard's rows are short: one segment per row when they span at most four
  // tiles (fewer, longer CTAs; measured 56 against 66 us for rank 0 of 8 on
  // 256 x 5 rows of 151936 bf16 entries)
  if (f.tiles <= 4) f.nseg = 1;
  // Draw CTAs of a shard take their sequence's decision before the race, so
  // one wave of them: chunks per sequence = draw slots / B, at least one and
  // at most one per 8 groups (f.nc2 <= lay.nc2).
  {
    const long long ng = (Vs + kRaceGroup - 1) / kRaceGroup;
    const long long slots = static_cast<long long>(sm_count()) * draw_ctas_per_sm(dtype == SV_BF16);
    const long long maxc = (ng + kDrawThreads / 32 - 1) / (kDrawThreads / 32);
    long long nc = slots / B;
    nc = nc < 1 ? 1 : (nc > maxc ? maxc : nc);
    f.gpc = static_cast<int>((ng + nc - 1) / nc);
    f.nc2 = static_cast<int>((ng + f.gpc - 1) / f.gpc);
  }
  f.voff = v0;
  f.vfull = V;
  if (static_cast<long long>(B) * f.nc2 > INT_MAX ||
      static_cast<long long>(B) * (gamma + 1) * f.nseg > INT_MAX)
    return set_error(SV_ERR_INVALID_ARG, "B x Vs too large for one launch");
  return SV_OK;
}
}  // namespace

int launch_shard_stats(const void* target, const void* draft, const int32_t* tokens,
                       const float* temps, int B, int gamma, int V, int v0, int Vs, int dtype,
                       void* out_stats, void* workspace, const Layout& lay, cudaStream_t stream) {
  SingleParams f{};
  int rc = shard_params(f, target, draft, tokens, temps, B, gamma, V, v0, Vs, dtype, 0, 0, nullptr,
                        nullptr, nullptr, nullptr, workspace, lay);
  if (rc != SV_OK) return rc;
  f.xstats = static_cast<float4*>(out_stats);
  const dim3 grid(static_cast<unsigned>(static_cast<long long>(B) * (gamma + 1) * f.nseg));
  const cudaError_t e = dtype == SV_BF16 ? launch_pdl(rows_kernel<true, true>, grid, kRowThreads, stream, f)
                                         : launch_pdl(rows_kernel<false, true>, grid, kRowThreads, stream, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "shard row kernel launch failed: %s", cudaGetErrorString(e));
  return check_launch("shard statistics");
}

int launch_shard_decide(const void* target, const void* draft, const int32_t* tokens,
                        const float* temps, int B, int gamma, int V, int v0, int Vs, int dtype,
                        const void* all_stats, int nshards, uint64_t seed, uint64_t step,
                        int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                        float* out_lq, void* out_candidate, void* workspace, const Layout& lay,
                        cudaStream_t stream) {
  SingleParams f{};
  int rc = shard_params(f, target, draft, tokens, temps, B, gamma, V, v0, Vs, dtype, seed, step,
                        out_accept_len, out_tokens, out_lp, out_lq, workspace, lay);
  if (rc != SV_OK) return rc;
  f.cand = static_cast<ShardCand*>(out_candidate);
  f.allstats = static_cast<const float4*>(all_stats);
  f.nshards = nshards;
  const dim3 grid2(static_cast<unsigned>(static_cast<long long>(B) * f.nc2));
  const cudaError_t e = dtype == SV_BF16 ? launch_pdl(draw_kernel<true, true>, grid2, kDrawThreads, stream, f)
                                         : launch_pdl(draw_kernel<false, true>, grid2, kDrawThreads, stream, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "shard draw kernel launch failed: %s", cudaGetErrorString(e));
  return check_launch("shard decide");
}

int launch_shard_pick(const void* all_candidates, int nshards, int B, int gamma,
                      int32_t* out_accept_len, int32_t* out_tokens, cudaStream_t stream) {
  constexpr int kPerBlock = kPickThreads / 32;  // sequences per CTA
  shard_pick_kernel<<<(B + kPerBlock - 1) / kPerBlock, kPickThreads, 0, stream>>>(
      static_cast<const ShardCand*>(all_candidates), nshards, B, gamma, out_accept_len, out_tokens);
  return check_launch("shard pick");
}

}  // namespace sv
