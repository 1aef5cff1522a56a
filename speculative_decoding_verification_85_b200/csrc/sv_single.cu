// sv_single.cu -- single-draft verification: one persistent kernel per call.
//
// What it computes (per sequence b with temperature T > 0): the
// temperature-scaled log-softmax of every needed row, the two
// log-probabilities of each draft token, the acceptance test
// u_i < min(1, p/q) with the first rejection j ("FlashSpec", Methodology
// s.1; "FlexDraft", Problem definition), and the correction token at j drawn
// from max(p_j - q_j, 0) or the bonus token from p_gamma ("Speculative
// Speculative Decoding", s.2 Saguaro sampling), as a Gumbel-max with Philox
// noise keyed per vocabulary entry.  T = 0 is greedy argmax matching.
//
// How: a grid of two CTAs per SM claims work items from a counter in the
// workspace, in a fixed order:
//   - row items: (sequence b, position i, vocabulary segment) -- target row i
//     and draft row i over the segment, streamed through a ring of shared-
//     memory stages by one-dimensional bulk copies (TMA) that a producer warp
//     issues, and reduced by eight consumer warps to the row maximum and an
//     integer-reference softmax sum; the CTA whose item completes a sequence
//     (arrival ticket) combines its partials and makes the decision, then
//     publishes it with a release flag;
//   - draw items: (sequence b, vocabulary chunk) -- the exponential race of
//     the correction/bonus draw over a strided part of the vocabulary.  A
//     sequence's draw items are queued `lag` sequences after its row items, so
//     the ALU-bound race of one sequence runs beside the HBM-bound rows of
//     later ones.  Philox is evaluated only for 4-entry blocks that can still
//     win: since E = -ln U > 2^-24 for every keyed uniform, a block whose
//     largest weight w satisfies w 2^24 <= (a lower bound of the winning ratio)
//     is skipped, exactly.  Skipped-or-not blocks are compacted per warp so
//     that Philox runs on full warps.
// A draw item waits (bounded) for its sequence's decision flag.  Items are
// claimed in queue order and every row item precedes the draw items that wait
// on it, so the item being waited on has been claimed by a running CTA, which
// processes its items in claim order and never waits on a later item: the
// waits always end.
#include <atomic>
#include <climits>

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"
#include "sv_stream.cuh"

namespace sv {

// ------------------------------------------------------------------ decision
// Acceptance probability min(1, p/q) from log-probabilities (fp64); q = 0
// accepts when p > 0, 0/0 rejects.
__device__ __forceinline__ double accept_prob(double lp, double lq) {
  if (lq == -INFINITY) return lp == -INFINITY ? 0.0 : 1.0;
  const double r = exp(lp - lq);
  return r < 1.0 ? r : 1.0;
}

// Warp 0 of the CTA that completed sequence b: validate, accept/reject, write
// outputs, publish the draw's hand-off record and raise the sequence's
// decision flag (1 + mode, release).  T is the sequence's temperature and
// x[0..gamma) its draft tokens (staged in shared memory by the caller).
template <bool kBf16>
__device__ __noinline__ void decide_single(const CallParams& p, int b, float T, const int* x,
                                           const RowAcc* rows, const float* zsel,
                                           unsigned* ready) {
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
    for (int i = lane; i <= g; i += 32) tok[i] = -1;
    for (int i = lane; i < g; i += 32) {
      if (p.out_lp) p.out_lp[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
      if (p.out_lq) p.out_lq[static_cast<size_t>(b) * g + i] = __int_as_float(0x7fc00000);
    }
    if (lane == 0) {
      p.accept_len[b] = -1;
      p.info[b].mode = kModeNone;
      st_release(ready + b, 1u + kModeNone);
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
        const RowAcc& ap = rows[i];
        const RowAcc& aq = rows[g + 1 + i];
        // d = fl32(fl32(z_x / T) - fl32(zmax / T)): the same fp32 operations
        // as scaling the whole row and shifting by its maximum; the draft
        // token's logits were picked up while the rows streamed
        const float dp = __fsub_rn(__fdiv_rn(zsel[2 * i], T), __fdiv_rn(ap.m, T));
        const float dq = __fsub_rn(__fdiv_rn(zsel[2 * i + 1], T), __fdiv_rn(aq.m, T));
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
      si.lsp = log2f(rows[j].s);
      if (j < g) {
        si.zmq = rows[g + 1 + j].m;
        si.lsq = log2f(rows[g + 1 + j].s);
      }
    }
    p.info[b] = si;
    st_release(ready + b, 1u + static_cast<unsigned>(si.mode));  // after the record
  }
}

// ------------------------------------------------------------------ layout
constexpr int kCWarps = 8;                     // consumer warps of a CTA
constexpr int kCThreads = 32 * kCWarps;        // 256 consumer threads
constexpr int kVThreads = kCThreads + 32;      // + one producer warp
constexpr int kStages = 3;                     // shared-memory ring stages
constexpr int kSlotBytes = kTileVec * 16;      // one row's tile: 16 KB
constexpr int kStageBytes = 2 * kSlotBytes;    // target tile + draft tile
constexpr int kRingBytes = kStages * kStageBytes;
constexpr int kQCap = 64;                      // per-warp race queue (power of two)
constexpr int kRaceRound = kCThreads;          // Philox blocks per CTA per race round
static_assert(kCThreads == kTileThreads, "one consumer thread per tile lane");

enum ItemKind : int { kItemEnd = 0, kItemRow = 1, kItemDraw = 2 };
constexpr int kFirstTile = 1, kLastTile = 2;

// What the producer hands the consumers with each ring stage.
struct alignas(16) TileDesc {
  int kind;   // ItemKind
  int b;      // sequence
  int i;      // position (row item) or chunk (draw item)
  int seg;    // vocabulary segment (row item)
  int kb;     // first body vector of the tile (row item)
  int nvA;    // 16-byte vectors of the target tile in the stage (0: not read)
  int nvB;    // vectors of the draft tile (0: not read)
  int flags;  // kFirstTile | kLastTile
  float T;    // the sequence's temperature
  int xg;     // the draft token at i (softmax rows with i < gamma), else -1
  int pad0, pad1;
};

struct SingleParams {
  CallParams p1;       // inputs, outputs, row arrivals (ticket), hand-off (info)
  float4* pairpart;     // [B][gamma + 1][nseg] x {target, draft} partials
  float* zx;            // [B][gamma][nseg][2] draft token's target / draft logit
  RacePartial* part2;   // [B][nd] draw partials
  unsigned* ticket2;    // [B] draw arrivals
  unsigned* ready;      // [B] decision flags (1 + mode once decided)
  unsigned* bar;        // [B] draw bars (float bits, monotone)
  unsigned* ctl;        // control words (kCtlNext, kCtlExit, kCtlError)
  int nseg;             // row segments per row
  int segvec;           // 16-byte vectors per row segment (multiple of kTileVec)
  int nd;               // draw items per sequence
  int nr;               // row items per sequence: (gamma + 1) nseg
  int lag;              // sequences between a sequence's rows and its draw items
  int total;            // items in the queue: B (nr + nd)
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

// Item at queue position q: the row items of the first `lag` sequences, then
// for k = 0, 1, ... the row items of sequence lag + k followed by the draw
// items of sequence k, then the remaining draw items.
struct Item {
  int kind, b, idx;  // idx: row item within the sequence (i nseg + seg), or draw chunk
};
__device__ __forceinline__ Item decode_item(const SingleParams& f, int q) {
  const int nr = f.nr, nd = f.nd, lag = f.lag, B = f.p1.B;
  if (q < lag * nr) return Item{kItemRow, q / nr, q % nr};
  q -= lag * nr;
  const int mid = B - lag;
  if (q < mid * (nr + nd)) {
    const int k = q / (nr + nd), r = q % (nr + nd);
    return r < nr ? Item{kItemRow, lag + k, r} : Item{kItemDraw, k, r - nr};
  }
  q -= mid * (nr + nd);
  return Item{kItemDraw, mid + q / nd, q % nd};
}

// ------------------------------------------------------------ shared memory
struct alignas(16) VerifySmem {
  TileDesc desc[kStages];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  RowAcc rows[kMaxRowsPerSeq];
  RowAcc scratch[2 * kCWarps];
  float2 zxw[kCWarps];
  float zsel[2 * SV_MAX_GAMMA];
  int tok[SV_MAX_GAMMA];
  float4 race[kCWarps];
  float4 qw[kCWarps][kQCap];  // race queue: weights of a pending block
  int qg[kCWarps][kQCap];     // race queue: the pending block
  SeqInfo info;
  int last;
};

// ---------------------------------------------------------------- producer
// Lane 0 of the producer warp: claim items (one ahead), describe each ring
// stage and issue its bulk copies.  Rows are read from the first 16-byte
// boundary on; the unaligned head and tail of a row are read by the
// consumers as scalars.
template <bool kBf16>
__device__ void produce(const SingleParams& f, VerifySmem& sm, char* ring) {
  const CallParams& p = f.p1;
  unsigned* next = f.ctl + kCtlNext;
  int stage = 0;
  uint32_t phase = 1;  // a fresh barrier's preceding phase counts as complete
  auto take = [&](TileDesc& d) -> bool {
    if (!mbar_wait(&sm.empty[stage], phase)) {
      atomicExch(f.ctl + kCtlError, 1u);
      return false;
    }
    sm.desc[stage] = d;
    return true;
  };
  auto advance = [&]() {
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1u;
    }
  };
  int cur = static_cast<int>(atomicAdd(next, 1u));
  for (;;) {
    const int nxt = cur < f.total ? static_cast<int>(atomicAdd(next, 1u)) : 0;
    if (cur >= f.total) {
      TileDesc d{};
      d.kind = kItemEnd;
      if (take(d)) mbar_arrive(&sm.full[stage]);
      return;
    }
    const Item it = decode_item(f, cur);
    TileDesc d{};
    d.b = it.b;
    if (it.kind == kItemDraw) {
      d.kind = kItemDraw;
      d.i = it.idx;
      if (!take(d)) return;
      mbar_arrive(&sm.full[stage]);
      advance();
    } else {
      const int i = it.idx / f.nseg, seg = it.idx - i * f.nseg;
      const float T = __ldg(p.temps + it.b);
      const int modeA = row_mode(T, true);
      const bool loadA = modeA != kRowSkip;
      const bool loadB = i < p.gamma && row_mode(T, false) == kRowLse;
      int xg = -1;
      if (modeA == kRowLse && i < p.gamma) {
        const int xt = __ldg(p.tokens + static_cast<size_t>(it.b) * p.gamma + i);
        if (xt >= 0 && xt < p.V) xg = xt;
      }
      const char* rpA = target_row<kBf16>(p, it.b, i);
      const char* rpB = loadB ? draft_row<kBf16>(p, it.b, i) : rpA;
      const RowGeom<kBf16> gA(rpA, p.V), gB(rpB, p.V);
      const int k0 = seg * f.segvec;
      const int a1 = loadA ? min(gA.nvec, k0 + f.segvec) : k0;
      const int b1 = loadB ? min(gB.nvec, k0 + f.segvec) : k0;
      const int kend = max(max(a1, b1), k0 + 1);  // at least one stage per item
      d.kind = kItemRow;
      d.i = i;
      d.seg = seg;
      d.T = T;
      d.xg = xg;
      const uint4* vA = gA.body(rpA);
      const uint4* vB = gB.body(rpB);
      for (int kb = k0; kb < kend; kb += kTileVec) {
        d.kb = kb;
        d.nvA = max(0, min(a1 - kb, kTileVec));
        d.nvB = max(0, min(b1 - kb, kTileVec));
        d.flags = (kb == k0 ? kFirstTile : 0) | (kb + kTileVec >= kend ? kLastTile : 0);
        if (!take(d)) return;
        const uint32_t bytes = static_cast<uint32_t>(d.nvA + d.nvB) * 16u;
        char* st = ring + stage * kStageBytes;
        if (bytes) {
          mbar_arrive_expect_tx(&sm.full[stage], bytes);
          if (d.nvA) bulk_g2s(st, vA + kb, static_cast<uint32_t>(d.nvA) * 16u, &sm.full[stage]);
          if (d.nvB)
            bulk_g2s(st + kSlotBytes, vB + kb, static_cast<uint32_t>(d.nvB) * 16u, &sm.full[stage]);
        } else {
          mbar_arrive(&sm.full[stage]);
        }
        advance();
      }
    }
    cur = nxt;
  }
}

// --------------------------------------------------------- row reductions
__device__ __forceinline__ RowAcc empty_lse_acc() {
  return RowAcc{-INFINITY, 0.0f, __float_as_int(-INFINITY), 0};
}
__device__ __forceinline__ RowAcc empty_argmax_acc() { return RowAcc{-INFINITY, 0.0f, 0x7fffffff, 0}; }

__device__ __forceinline__ float first_number(float z) {  // any lane's non-NaN value
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, z, off);
    if (z != z) z = o;
  }
  return z;
}

// Consumer-wide reduction of the two rows' accumulators and of the draft
// token's two picked-up logits: a butterfly within each warp, then warp 0
// merges the 8 warp results of each row by a 3-step butterfly (lanes 0-7 row
// A, lanes 8-15 row B).  One barrier; the result is valid in thread 0.
__device__ __forceinline__ void reduce_pair(RowAcc& A, RowAcc& B, float2& z, bool argmaxA,
                                            VerifySmem& sm) {
  constexpr int W = kCWarps;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  warp_merge(A, argmaxA);
  warp_merge(B, false);
  z.x = first_number(z.x);
  z.y = first_number(z.y);
  if (lane == 0) {
    sm.scratch[warp] = A;
    sm.scratch[W + warp] = B;
    sm.zxw[warp] = z;
  }
  block_sync<kCThreads>();
  if (warp == 0) {
    const bool rowB = lane >= W;
    RowAcc v = lane < 2 * W ? sm.scratch[lane] : empty_lse_acc();
    group_merge<W>(v, rowB ? false : argmaxA);
    const RowAcc vb = shfl_xor_acc(v, W);  // lane 0 receives lane 8's row-B result
    if (lane == 0) {
      A = v;
      B = vb;
      for (int w = 0; w < W; ++w) {
        const float2 q = sm.zxw[w];
        if (q.x == q.x) z.x = q.x;
        if (q.y == q.y) z.y = q.y;
      }
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

// Combine the nseg segment partials of every position of sequence b into the
// row table sm.rows (target rows 0..gamma, then draft rows), and pick up the
// draft tokens' logits (sm.zsel[2i], [2i + 1]).
__device__ __forceinline__ void combine_pairs(const SingleParams& f, int b, bool argmaxA, float c,
                                              VerifySmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = f.p1.gamma;
  for (int i = warp; i <= g; i += kCWarps) {
    RowAcc A = argmaxA ? empty_argmax_acc() : empty_lse_acc(), B = empty_lse_acc();
    float zt = __int_as_float(0x7fc00000), zd = zt;
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
    zt = first_number(zt);
    zd = first_number(zd);
    if (lane == 0) {
      if (!argmaxA) A.s = sum_rel_max(A, c);
      B.s = sum_rel_max(B, c);
      sm.rows[i] = A;
      if (i < g) {
        sm.rows[g + 1 + i] = B;
        sm.zsel[2 * i] = zt;
        sm.zsel[2 * i + 1] = zd;
      }
    }
  }
  block_sync<kCThreads>();
}

// Head (entries before the first 16-byte boundary) and tail (after the last)
// of a row, read as scalars by the first / last segment's item.
template <bool kBf16>
__device__ __forceinline__ void row_edges(const char* rp, int V, const RowGeom<kBf16>& g, bool argmax,
                                          float c, bool head, bool tail, int xg, float& zx,
                                          RunAcc& acc) {
  const int tid = threadIdx.x;
  if (head)
    for (int v = tid; v < g.head; v += kCThreads) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) zx = z;
      if (argmax) argmax_scalar(acc, z, v); else lse_scalar(acc, z, c);
    }
  if (tail)
    for (int v = g.tail0 + tid; v < V; v += kCThreads) {
      const float z = logit_at<kBf16>(rp, v);
      if (v == xg) zx = z;
      if (argmax) argmax_scalar(acc, z, v); else lse_scalar(acc, z, c);
    }
}

// The body vector that holds entry xg of a row, if this thread loads it within
// the segment [k0, k1); -1 otherwise.  Tiles start at k0 + t kTileVec, so the
// thread that loads vector k is (k - k0) mod kCThreads in every tile.
template <bool kBf16>
__device__ __forceinline__ int owned_vector(const RowGeom<kBf16>& g, int xg, int k0, int k1) {
  if (xg < g.head || xg >= g.tail0) return -1;
  const int k = (xg - g.head) / Vec16<kBf16>::kN;
  if (k < k0 || k >= k1 || (k - k0) % kCThreads != static_cast<int>(threadIdx.x)) return -1;
  return k;
}

template <bool kBf16>
__device__ __forceinline__ void pick_logit(const uint4 (&r)[kTileRegs], int own, int kb, int xg,
                                           const RowGeom<kBf16>& g, float& zx) {
  if (own < kb || own >= kb + kTileVec) return;
  const int j = (own - kb) / kCThreads;
  const int e = (xg - g.head) % Vec16<kBf16>::kN;
#pragma unroll
  for (int q = 0; q < kTileRegs; ++q)  // compile-time q keeps r[] in registers
    if (q == j) zx = Vec16<kBf16>::at(r[q], e);
}

// The thread's vectors of a staged tile (nv valid vectors); the rest read as -inf.
template <bool kBf16>
__device__ __forceinline__ void stage_tile(const char* slot, int nv, uint4 (&r)[kTileRegs]) {
  constexpr uint32_t ninf = Vec16<kBf16>::kNegInf;
  const uint4* v = reinterpret_cast<const uint4*>(slot);
#pragma unroll
  for (int j = 0; j < kTileRegs; ++j) {
    const int k = static_cast<int>(threadIdx.x) + j * kCThreads;
    r[j] = k < nv ? lds128(v + k) : make_uint4(ninf, ninf, ninf, ninf);
  }
}

// ------------------------------------------------------------------- races
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
  __device__ __forceinline__ float at(int w) const {
    return w == 0 ? r.x : (w == 1 ? r.y : (w == 2 ? r.z : r.w));
  }
  __device__ __forceinline__ void set_neg_inf() { r = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY); }
};

// Running winner of an exponential race: best weight / exponential pair and
// index, and a slightly lowered lower bound of the winning ratio for the
// cheap pre-tests.
struct Race {
  float bw, be;
  int bi;
  float lo;  // at most (winning ratio) (1 - 2^-20)
  __device__ __forceinline__ void reset() {
    bw = 0.0f;
    be = 1.0f;
    bi = INT_MAX;
    lo = 0.0f;
  }
  // Exact test of candidate v (weight w > 0, Philox word x).
  __device__ __forceinline__ void offer(float w, uint32_t x, int v) {
    const float e = exponential_from_bits(x);
    if (race_better(w, e, v, bw, be, bi)) {
      bw = w;
      be = e;
      bi = v;
      lo = fmaxf(lo, __fdiv_rn(bw, be) * (1.0f - 0x1p-20f));
    }
  }
};

// Candidates of one Philox block (entries v0 .. v0 + 3).  First a bound
// without logarithms: since -ln U <= (1 - U) / U, every candidate's ratio
// w / E is at least w U / t (t = 1 - U), so the block's largest such bound
// (lowered for rounding) is a valid bar.  Then every entry runs the cheap
// test w > lo t: since E >= t, w / t must beat the bar (lowered, so the test
// never drops a possible winner; with lo >= 0 it also rejects w <= 0).  Only
// entries that pass take the logarithm.
__device__ __forceinline__ void race_block(Race& race, const float4& wv, const uint4& rnd, int v0) {
  const float w[4] = {wv.x, wv.y, wv.z, wv.w};
  float t[4];
  float lb = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t[k] = gumbel_one_minus_u(word_of(rnd, k));
    lb = fmaxf(lb, __fdividef(w[k] * (1.0f - t[k]), t[k]));
  }
  race.lo = fmaxf(race.lo, lb * (1.0f - 0x1p-20f));
  bool pass[4];
  bool any = false;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    pass[k] = w[k] > race.lo * t[k];
    any |= pass[k];
  }
  if (any) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (pass[k] && w[k] > 0.0f) race.offer(w[k], word_of(rnd, k), v0 + k);
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Exponential race of sequence b's draw over the Philox blocks of chunk
// `chunk` of nchunk (round r covers blocks [(r nchunk + chunk) 256, + 256);
// warp w takes 32 of them): the winner of w_v / E_v (E_v = -ln U_v) with
// w = max(p - q, 0) (residual) or w = p (bonus), p_v = 2^{(z_v - zmp) c - lsp}.
// A block is queued for Philox only if 2^24 max_k w_k exceeds the warp's bar
// (exact: E > 2^-24, so a skipped entry's ratio stays below the bar, which is
// below the winning ratio); the queue is flushed 32 blocks at a time, so
// Philox runs on full warps.  `gbar` (or NULL) is the sequence's shared bar:
// read every few rounds, raised when this warp's bar grows.
template <bool kBf16>
__device__ void race_chunk(const SingleParams& f, const SeqInfo& si, int b, int chunk, int nchunk,
                           unsigned* gbar, Race& race, VerifySmem& sm) {
  constexpr uintptr_t kVecAlign = kBf16 ? 8 : 16;
  const CallParams& p = f.p1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const char* trow = target_row<kBf16>(p, b, si.j);
  const bool resid = si.mode == kModeResidual;
  const char* drow = resid ? draft_row<kBf16>(p, b, si.j) : trow;
  const bool tvec = (reinterpret_cast<uintptr_t>(trow) % kVecAlign) == 0;
  const bool dvec = (reinterpret_cast<uintptr_t>(drow) % kVecAlign) == 0;
  const float2 nm = make_float2(-si.zmp, -si.zmq), cc = make_float2(si.c, si.c),
               nl = make_float2(-si.lsp, -si.lsq);
  const PhiloxStream ps(p.seed, p.step, kTagGumbel, b, 0, si.j);
  const int nblocks = (p.V + 3) / 4;
  float4* qw = sm.qw[warp];
  int* qg = sm.qg[warp];
  int qh = 0, qn = 0;  // queue head and length (warp-uniform)
  float published = 0.0f;
  unsigned gnext = 0;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (gbar && lane == 0) gnext = ld_relaxed(gbar);
  for (int r = 0;; ++r) {
    const int base = (r * nchunk + chunk) * kRaceRound;
    if (base >= nblocks) break;  // uniform over the CTA
    const int g = base + warp * 32 + lane;
    float w[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (g < nblocks) {
      Block4<kBf16> t, d;
      t.load(trow, tvec, p.V, g);
      if (resid) d.load(drow, dvec, p.V, g); else d.set_neg_inf();
      // p_v = 2^{(z_v - zmp) c - lsp}, q_v likewise: the target and draft
      // value of an entry travel as one packed pair
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 e = __ffma2_rn(__fadd2_rn(make_float2(t.at(k), d.at(k)), nm), cc, nl);
        w[k] = ex2_approx(e.x);
        if (resid) w[k] -= ex2_approx(e.y);
      }
    }
    if (gbar) {  // the shared bar read one round earlier
      const float gv = __uint_as_float(__shfl_sync(0xffffffffu, gnext, 0));
      race.lo = fmaxf(race.lo, gv);
      if (lane == 0 && (r & 3) == 3) gnext = ld_relaxed(gbar);
    }
    const float wm = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
    const bool need = wm * 16777216.0f > race.lo;
    const unsigned bal = __ballot_sync(0xffffffffu, need);
    if (bal == 0xffffffffu && qn == 0) {
      race_block(race, make_float4(w[0], w[1], w[2], w[3]), ps.block(g), 4 * g);
    } else if (bal) {
      const int pos = (qh + qn + __popc(bal & lt_mask)) & (kQCap - 1);
      if (need) {
        qw[pos] = make_float4(w[0], w[1], w[2], w[3]);
        qg[pos] = g;
      }
      qn += __popc(bal);
      __syncwarp();
      if (qn >= 32) {
        const int e = (qh + lane) & (kQCap - 1);
        const float4 ww = qw[e];
        const int gg = qg[e];
        qh = (qh + 32) & (kQCap - 1);
        qn -= 32;
        __syncwarp();  // entries read before later rounds overwrite them
        race_block(race, ww, ps.block(gg), 4 * gg);
      }
    }
    race.lo = warp_max(race.lo);
    if (gbar && lane == 0 && race.lo > 2.0f * published) {
      atomicMax(gbar, __float_as_uint(race.lo));  // non-negative floats order as their bits
      published = race.lo;
    }
  }
  if (qn > 0) {  // the rest of the queue
    const int e = (qh + lane) & (kQCap - 1);
    const float4 ww = lane < qn ? qw[e] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const int gg = lane < qn ? qg[e] : 0;
    __syncwarp();
    if (lane < qn) race_block(race, ww, ps.block(gg), 4 * gg);
  }
}

// --------------------------------------------------------------- consumers
// Bounded wait for sequence b's decision flag (thread 0).  Returns the flag,
// or 0 when the wait ran out of time (then the kernel's error word is set).
__device__ __forceinline__ unsigned wait_decision(const SingleParams& f, int b) {
  unsigned v = ld_acquire(f.ready + b);
  if (v) return v;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(it < 64 ? 32 : 128);
    v = ld_acquire(f.ready + b);
    if (v) return v;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  atomicExch(f.ctl + kCtlError, 2u);
  return 0;
}

// A draw item: chunk `chunk` of sequence b's race, and, in the CTA that
// completes the sequence's draw items, the combined winner (the token) and
// the reset of the sequence's flags for the next call.
template <bool kBf16>
__device__ void draw_item(const SingleParams& f, int b, int chunk, VerifySmem& sm) {
  const CallParams& p = f.p1;
  const int tid = threadIdx.x;
  if (tid == 0) {
    const unsigned flag = wait_decision(f, b);
    SeqInfo si{};
    if (flag) {
      const float4* ip = reinterpret_cast<const float4*>(p.info + b);
      const float4 w0 = __ldcg(ip), w1 = __ldcg(ip + 1);
      si.mode = __float_as_int(w0.x);
      si.j = __float_as_int(w0.y);
      si.zmp = w0.z;
      si.zmq = w0.w;
      si.c = w1.x;
      si.lsp = w1.y;
      si.lsq = w1.z;
    } else {
      si.mode = kModeNone;  // the decision never came: mark the sequence invalid
      p.accept_len[b] = -1;
      for (int i = 0; i <= p.gamma; ++i) p.out_tokens[static_cast<size_t>(b) * (p.gamma + 1) + i] = -1;
    }
    sm.info = si;
  }
  block_sync<kCThreads>();
  const SeqInfo si = sm.info;
  const bool draw = (si.mode == kModeResidual && si.j >= 0 && si.j < p.gamma) ||
                    (si.mode == kModeBonus && si.j == p.gamma);
  Race race;
  race.reset();
  if (draw) {
    // bonus draw: the entry at the row maximum has weight 2^-lsp and E < 17,
    // so its ratio -- and the winner's -- exceeds 2^-lsp / 17
    if (si.mode == kModeBonus) race.lo = ex2_approx(-si.lsp) * (1.0f / 17.0f);
    race_chunk<kBf16>(f, si, b, chunk, f.nd, f.bar + b, race, sm);
  }
  float bw = race.bw, be = race.be;
  int bi = race.bi;
  race_reduce<kCThreads>(bw, be, bi, sm.race);
  if (tid == 0) {
    RacePartial* pp = f.part2 + static_cast<size_t>(b) * f.nd + chunk;
    *reinterpret_cast<float4*>(pp) = make_float4(bw, be, __int_as_float(bi), 0.0f);
    const unsigned t = ticket_acq_rel(f.ticket2 + b);
    sm.last = (t == static_cast<unsigned>(f.nd - 1));
  }
  block_sync<kCThreads>();  // orders the other threads after thread 0's acquire
  if (!sm.last) return;
  if (draw) {
    bw = 0.0f;
    be = 1.0f;
    bi = INT_MAX;
    for (int q = tid; q < f.nd; q += kCThreads) {
      const float4 g = __ldcg(reinterpret_cast<const float4*>(f.part2 + static_cast<size_t>(b) * f.nd + q));
      if (race_better(g.x, g.y, __float_as_int(g.z), bw, be, bi)) {
        bw = g.x;
        be = g.y;
        bi = __float_as_int(g.z);
      }
    }
    race_reduce<kCThreads>(bw, be, bi, sm.race);
    if (!(bw > 0.0f)) {  // uniform: race_reduce returns the winner to every thread
      // the residual vanished (p_j == q_j to rounding): draw from p_j instead,
      // over the whole row in this CTA (without the residual race's bar)
      SeqInfo sb = si;
      sb.mode = kModeBonus;
      race.reset();
      race.lo = ex2_approx(-sb.lsp) * (1.0f / 17.0f);
      race_chunk<kBf16>(f, sb, b, 0, 1, nullptr, race, sm);
      bw = race.bw;
      be = race.be;
      bi = race.bi;
      race_reduce<kCThreads>(bw, be, bi, sm.race);
    }
    if (tid == 0) p.out_tokens[static_cast<size_t>(b) * (p.gamma + 1) + si.j] = bi;
  }
  if (tid == 0) {  // every chunk of b is past its wait and its race
    f.ready[b] = 0u;
    f.bar[b] = 0u;
    f.ticket2[b] = 0u;
  }
}

// Per-item state of a row item, set up at its first tile.
template <bool kBf16>
struct RowItem {
  int b, i, seg;
  float T, c;
  bool argmaxA, loadA, loadB;
  int xg, ownA, ownB;
  const char* rpA;
  const char* rpB;
  RowGeom<kBf16> gA, gB;
  __device__ __forceinline__ RowItem(const SingleParams& f, const TileDesc& d)
      : b(d.b), i(d.i), seg(d.seg), T(d.T), xg(d.xg),
        rpA(target_row<kBf16>(f.p1, d.b, d.i)),
        rpB(d.i < f.p1.gamma ? draft_row<kBf16>(f.p1, d.b, d.i) : rpA),
        gA(rpA, f.p1.V), gB(rpB, f.p1.V) {
    const int modeA = row_mode(T, true);
    argmaxA = modeA == kRowArgmax;
    loadA = modeA != kRowSkip;
    loadB = i < f.p1.gamma && row_mode(T, false) == kRowLse;
    c = modeA == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
    const int k0 = seg * f.segvec;
    ownA = owned_vector<kBf16>(gA, xg, k0, min(gA.nvec, k0 + f.segvec));
    ownB = owned_vector<kBf16>(gB, xg, k0, min(gB.nvec, k0 + f.segvec));
  }
};

// The end of a row item: row edges, the consumer-wide reduction, the partial
// and the arrival ticket; the CTA that completes the sequence decides.
template <bool kBf16>
__device__ void row_item_end(const SingleParams& f, const RowItem<kBf16>& it, RunAcc& accA, RunAcc& accB,
                             float2 z, VerifySmem& sm) {
  const CallParams& p = f.p1;
  const int tid = threadIdx.x;
  const bool first = it.seg == 0, last = it.seg == f.nseg - 1;
  if (it.loadA && (first || last))
    row_edges<kBf16>(it.rpA, p.V, it.gA, it.argmaxA, it.c, first, last, it.xg, z.x, accA);
  if (it.loadB && (first || last))
    row_edges<kBf16>(it.rpB, p.V, it.gB, false, it.c, first, last, it.xg, z.y, accB);
  RowAcc A = it.argmaxA ? accA.argmax_row() : accA.lse_row(), B = accB.lse_row();
  reduce_pair(A, B, z, it.argmaxA, sm);
  if (tid == 0) {
    float4* pp = f.pairpart + ((static_cast<size_t>(it.b) * (p.gamma + 1) + it.i) * f.nseg + it.seg) * 2;
    pp[0] = make_float4(A.m, A.s, __int_as_float(A.arg), __int_as_float(A.bad));
    pp[1] = make_float4(B.m, B.s, __int_as_float(B.arg), __int_as_float(B.bad));
    if (it.i < p.gamma) {
      float* zz = f.zx + ((static_cast<size_t>(it.b) * p.gamma + it.i) * f.nseg + it.seg) * 2;
      zz[0] = z.x;
      zz[1] = z.y;
    }
    // release this item's partial; the last arriver also acquires the others'
    const unsigned tk = ticket_acq_rel(p.ticket + it.b);
    const unsigned arrivals = static_cast<unsigned>(f.nr);
    sm.last = (tk == arrivals - 1);
    if (sm.last) p.ticket[it.b] = 0;  // leave the counter at zero for the next call
  }
  block_sync<kCThreads>();  // orders the other threads after thread 0's acquire
  if (!sm.last) return;
  for (int k = tid; k < p.gamma; k += kCThreads)
    sm.tok[k] = __ldg(p.tokens + static_cast<size_t>(it.b) * p.gamma + k);
  combine_pairs(f, it.b, it.argmaxA, it.c, sm);  // ends with a consumer barrier
  if (tid < 32) decide_single<kBf16>(p, it.b, it.T, sm.tok, sm.rows, sm.zsel, f.ready);
  block_sync<kCThreads>();  // sm.rows / sm.tok are reused by the next decision
}

template <bool kBf16>
__device__ void consume(const SingleParams& f, VerifySmem& sm, const char* ring) {
  const int tid = threadIdx.x;
  int stage = 0;
  uint32_t phase = 0;
  RunAcc accA, accB;
  accA.reset();
  accB.reset();
  float2 z = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
  // the current row item (rebuilt at each item's first tile)
  RowItem<kBf16> it(f, TileDesc{kItemRow, 0, 0, 0, 0, 0, 0, 0, 0.0f, -1, 0, 0});
  for (;;) {
    if (!mbar_wait(&sm.full[stage], phase)) {
      if (tid == 0) atomicExch(f.ctl + kCtlError, 3u);
      return;
    }
    const TileDesc d = sm.desc[stage];
    if (d.kind == kItemEnd) return;
    const char* st = ring + stage * kStageBytes;
    if (d.kind == kItemDraw) {
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&sm.empty[stage]);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
      draw_item<kBf16>(f, d.b, d.i, sm);
      continue;
    }
    if (d.flags & kFirstTile) {
      it = RowItem<kBf16>(f, d);
      accA.reset();
      accB.reset();
      z = make_float2(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    }
    uint4 ra[kTileRegs], rb[kTileRegs];
    stage_tile<kBf16>(st, d.nvA, ra);
    stage_tile<kBf16>(st + kSlotBytes, d.nvB, rb);
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(&sm.empty[stage]);  // the stage may be refilled
    if (++stage == kStages) { stage = 0; phase ^= 1u; }
    if (d.nvA) {
      pick_logit<kBf16>(ra, it.ownA, d.kb, it.xg, it.gA, z.x);
      if (it.argmaxA)
        argmax_tile<kBf16>(accA, ra, it.gA.head + (d.kb + tid) * Vec16<kBf16>::kN);
      else
        lse_tile<kBf16>(accA, ra, it.c);
    }
    if (d.nvB) {
      pick_logit<kBf16>(rb, it.ownB, d.kb, it.xg, it.gB, z.y);
      lse_tile<kBf16>(accB, rb, it.c);
    }
    if (d.flags & kLastTile) row_item_end<kBf16>(f, it, accA, accB, z, sm);
  }
}

// --------------------------------------------------------------- the kernel
template <bool kBf16>
__global__ void __launch_bounds__(kVThreads, 2) verify_kernel(const __grid_constant__ SingleParams f) {
  extern __shared__ __align__(128) char ring[];
  __shared__ VerifySmem sm;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kCWarps);
    }
    mbar_init_fence();
  }
  __syncthreads();
  // the previous grid in the stream has completed (programmatic dependent
  // launch); the next may start launching its CTAs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  if (tid >= kCThreads) {
    if (tid == kCThreads) produce<kBf16>(f, sm, ring);
    return;
  }
  consume<kBf16>(f, sm, ring);
  block_sync<kCThreads>();
  if (tid == 0) {
    // the last CTA to leave returns the work counter to zero for the next call
    const unsigned t = ticket_acq_rel(f.ctl + kCtlExit);
    if (t == gridDim.x - 1) {
      f.ctl[kCtlNext] = 0u;
      f.ctl[kCtlExit] = 0u;
    }
  }
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

int draw_chunks(int V, int dtype) {  // upper bound on draw items per sequence
  (void)dtype;
  const int nb = (V + 3) / 4;
  return (nb + kRaceRound - 1) / kRaceRound;
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

// Opt the kernel into its dynamic shared memory (once per device) and return
// its resident CTAs per SM (0 if the attribute could not be set).
template <typename Kernel>
int prepare(Kernel kernel) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingBytes) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kVThreads, kRingBytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

int ctas_per_sm(bool bf16) {
  static std::atomic<int> slots[2][64];
  return bf16 ? per_device(slots[1], -1, [](int) { return prepare(verify_kernel<true>); })
              : per_device(slots[0], -1, [](int) { return prepare(verify_kernel<false>); });
}

template <typename K>
cudaError_t launch_pdl(K kernel, unsigned grid, cudaStream_t stream, const SingleParams& f) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kVThreads);
  cfg.dynamicSmemBytes = kRingBytes;
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
}  // namespace

int launch_single(const void* target, const void* draft, const int32_t* tokens,
                  const float* temps, int B, int gamma, int V, int dtype, uint64_t seed,
                  uint64_t step, int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                  float* out_lq, void* workspace, const Layout& lay, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  const bool bf16 = dtype == SV_BF16;
  const int per_sm = ctas_per_sm(bf16);
  if (per_sm <= 0)
    return set_error(SV_ERR_CUDA, "verification kernel cannot be made resident (%d CTAs per SM)",
                     per_sm);
  SingleParams f{};
  CallParams& p1 = f.p1;
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
  f.pairpart = reinterpret_cast<float4*>(ws + lay.part1);
  f.zx = reinterpret_cast<float*>(ws + lay.resid);
  f.part2 = reinterpret_cast<RacePartial*>(ws + lay.part2);
  f.ticket2 = reinterpret_cast<unsigned*>(ws + lay.ticket2);
  f.ready = reinterpret_cast<unsigned*>(ws + lay.ready);
  f.bar = reinterpret_cast<unsigned*>(ws + lay.bar);
  f.ctl = reinterpret_cast<unsigned*>(ws + lay.ctl);
  const long long ctas = static_cast<long long>(sm_count()) * per_sm;

  // Row segments: whole tiles, at most kMaxSegTiles per item, about
  // kItemsPerCta row items per CTA for balance; balanced so that segments
  // differ by at most one tile.
  {
    constexpr int kMaxSegTiles = 4, kItemsPerCta = 4;
    const int tiles = body_tiles(V, dtype);
    const long long pairs = static_cast<long long>(B) * (gamma + 1);
    long long st = pairs * tiles / (kItemsPerCta * ctas);
    st = st < 1 ? 1 : (st > kMaxSegTiles ? kMaxSegTiles : st);
    int nseg = static_cast<int>((tiles + st - 1) / st);
    if (nseg > lay.nc) nseg = lay.nc;
    st = (tiles + nseg - 1) / nseg;
    f.nseg = nseg;
    f.segvec = static_cast<int>(st) * kTileVec;
  }
  // Draw items: about kDrawBlocks Philox blocks per consumer thread each.
  {
    constexpr int kDrawBlocks = 16;
    const long long nb = (V + 3) / 4;
    long long nd = (nb + static_cast<long long>(kDrawBlocks) * kRaceRound - 1) /
                   (static_cast<long long>(kDrawBlocks) * kRaceRound);
    const long long rounds = (nb + kRaceRound - 1) / kRaceRound;  // every chunk has a round
    if (nd > rounds) nd = rounds;
    if (nd < 1) nd = 1;
    if (nd > lay.nc2) nd = lay.nc2;
    f.nd = static_cast<int>(nd);
  }
  f.nr = (gamma + 1) * f.nseg;
  // Lag: two CTA-loads of row items between a sequence's rows and its draws.
  {
    long long lag = (2 * ctas + f.nr - 1) / f.nr;
    if (lag > B) lag = B;
    if (lag < 1) lag = 1;
    f.lag = static_cast<int>(lag);
  }
  const long long total = static_cast<long long>(B) * (f.nr + f.nd);
  if (total > INT_MAX / 2)
    return set_error(SV_ERR_INVALID_ARG, "B x V too large for one launch (%lld work items)", total);
  f.total = static_cast<int>(total);
  const unsigned grid = static_cast<unsigned>(total < ctas ? total : ctas);
  const cudaError_t e = bf16 ? launch_pdl(verify_kernel<true>, grid, stream, f)
                             : launch_pdl(verify_kernel<false>, grid, stream, f);
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "verification kernel launch failed: %s", cudaGetErrorString(e));
  return check_launch("verify");
}

}  // namespace sv
