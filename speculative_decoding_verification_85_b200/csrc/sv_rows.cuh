// sv_rows.cuh -- pass 1: one CTA streams one chunk of one logit row.
//
// Each logit element is read exactly once from HBM with 16-byte vector loads
// (bf16x8 / f32x4); a row's few unaligned leading and trailing elements are
// read as scalars.  Per row the pass produces what the acceptance test and
// the correction draw need: the raw maximum (NaN-propagating), the base-2
// scaled sum S = sum_v 2^{(z_v - max) log2(e) / T} (the softmax normaliser of
// z / T), and, for greedy rows, the first index of the maximum.
#pragma once

#include "sv_device.cuh"
#include "sv_internal.h"

namespace sv {

enum RowMode { kRowSkip = 0, kRowLse = 1, kRowArgmax = 2 };

__device__ __forceinline__ int row_mode(float T, bool is_target) {
  if (!(T >= 0.0f) || isinf(T)) return kRowSkip;  // invalid temperature: nothing to read
  if (T == 0.0f) return is_target ? kRowArgmax : kRowSkip;  // greedy: draft rows unused
  return kRowLse;
}

struct RowAcc {
  float m;   // running raw max (finite elements)
  float s;   // sum of 2^{(z - m) c}
  int arg;   // first index of m (argmax mode)
  int bad;   // saw NaN
};

template <int kMode>
__device__ __forceinline__ void acc_scalar(RowAcc& a, float z, int v, float c) {
  if (z != z) {
    a.bad = 1;
    return;
  }
  if constexpr (kMode == kRowLse) {
    if (z == -INFINITY) return;
    if (z > a.m) {
      a.s = (a.m == -INFINITY) ? 0.0f : a.s * ex2_approx((a.m - z) * c);
      a.m = z;
    }
    a.s += ex2_approx((z - a.m) * c);
  } else {
    if (z > a.m) {
      a.m = z;
      a.arg = v;
    }
  }
}

template <int kMode, int kN>
__device__ __forceinline__ void acc_vector(RowAcc& a, const float (&z)[kN], int v0, float c) {
  float vm = z[0];
#pragma unroll
  for (int e = 1; e < kN; ++e) vm = max_nan(vm, z[e]);
  if (vm != vm) {
    a.bad = 1;
    return;
  }
  if constexpr (kMode == kRowLse) {
    if (vm == -INFINITY) return;
    if (vm > a.m) {
      a.s = (a.m == -INFINITY) ? 0.0f : a.s * ex2_approx((a.m - vm) * c);
      a.m = vm;
    }
    float t = 0.0f;
#pragma unroll
    for (int e = 0; e < kN; ++e) t += ex2_approx((z[e] - a.m) * c);
    a.s += t;
  } else {
    if (vm > a.m) {
      a.m = vm;
#pragma unroll
      for (int e = kN - 1; e >= 0; --e)
        if (z[e] == vm) a.arg = v0 + e;
    }
  }
}

template <bool kBf16>
struct VecLoad;

template <>
struct VecLoad<true> {
  static constexpr int kN = 8;
  __device__ __forceinline__ static void decode(const uint4& r, float (&z)[8]) {
    z[0] = bf16_lo(r.x);
    z[1] = bf16_hi(r.x);
    z[2] = bf16_lo(r.y);
    z[3] = bf16_hi(r.y);
    z[4] = bf16_lo(r.z);
    z[5] = bf16_hi(r.z);
    z[6] = bf16_lo(r.w);
    z[7] = bf16_hi(r.w);
  }
};

template <>
struct VecLoad<false> {
  static constexpr int kN = 4;
  __device__ __forceinline__ static void decode(const uint4& r, float (&z)[4]) {
    z[0] = __uint_as_float(r.x);
    z[1] = __uint_as_float(r.y);
    z[2] = __uint_as_float(r.z);
    z[3] = __uint_as_float(r.w);
  }
};

// Scan chunk `chunk` of `nc` of one row.  Chunks split the 16-byte-aligned
// body of the row into equal runs of vectors; chunk 0 also takes the
// unaligned head, the last chunk the ragged tail.
template <bool kBf16, int kMode, int kThreads>
__device__ __forceinline__ void scan_chunk(RowAcc& a, const char* rp, int V, int chunk, int nc,
                                           float c) {
  constexpr int es = kBf16 ? 2 : 4;
  constexpr int kN = VecLoad<kBf16>::kN;
  constexpr int kUnroll = 4;
  const int tid = threadIdx.x;
  const uintptr_t addr = reinterpret_cast<uintptr_t>(rp);
  int head = static_cast<int>(((16u - (addr & 15u)) & 15u) / es);
  if (head > V) head = V;
  const int nvec = (V - head) / kN;
  const int tail0 = head + nvec * kN;
  const int cv = (nvec + nc - 1) / nc;
  const int k_begin = chunk * cv;
  const int k_end = min(nvec, k_begin + cv);

  if (chunk == 0)
    for (int v = tid; v < head; v += kThreads) acc_scalar<kMode>(a, logit_at<kBf16>(rp, v), v, c);

  const uint4* vp = reinterpret_cast<const uint4*>(rp + static_cast<size_t>(head) * es);
  for (int k0 = k_begin + tid; k0 < k_end; k0 += kUnroll * kThreads) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int k = k0 + u * kThreads;
      if (k < k_end) raw[u] = __ldg(vp + k);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int k = k0 + u * kThreads;
      if (k < k_end) {
        float z[kN];
        VecLoad<kBf16>::decode(raw[u], z);
        acc_vector<kMode>(a, z, head + k * kN, c);
      }
    }
  }

  if (chunk == nc - 1)
    for (int v = tail0 + tid; v < V; v += kThreads)
      acc_scalar<kMode>(a, logit_at<kBf16>(rp, v), v, c);
}

template <int kMode>
__device__ __forceinline__ void acc_merge(RowAcc& a, const RowAcc& o, float c) {
  a.bad |= o.bad;
  if constexpr (kMode == kRowLse) {
    lse_merge(a.m, a.s, o.m, o.s, c);
  } else {
    argmax_merge(a.m, a.arg, o.m, o.arg);
  }
}

// Block reduction to thread 0.  `scratch` holds kThreads / 32 entries.
template <int kMode, int kThreads>
__device__ __forceinline__ RowAcc block_reduce_acc(RowAcc a, float c, RowAcc* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    RowAcc o;
    o.m = __shfl_down_sync(0xffffffffu, a.m, off);
    o.s = __shfl_down_sync(0xffffffffu, a.s, off);
    o.arg = __shfl_down_sync(0xffffffffu, a.arg, off);
    o.bad = __shfl_down_sync(0xffffffffu, a.bad, off);
    acc_merge<kMode>(a, o, c);
  }
  if (lane == 0) scratch[warp] = a;
  block_sync<kThreads>();
  if (warp == 0) {
    constexpr int kWarps = kThreads / 32;
    a = lane < kWarps ? scratch[lane] : RowAcc{-INFINITY, 0.0f, 0x7fffffff, 0};
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      RowAcc o;
      o.m = __shfl_down_sync(0xffffffffu, a.m, off);
      o.s = __shfl_down_sync(0xffffffffu, a.s, off);
      o.arg = __shfl_down_sync(0xffffffffu, a.arg, off);
      o.bad = __shfl_down_sync(0xffffffffu, a.bad, off);
      acc_merge<kMode>(a, o, c);
    }
  }
  return a;
}

__device__ __forceinline__ void store_partial(RowPartial* p, const RowAcc& a) {
  *reinterpret_cast<float4*>(p) =
      make_float4(a.m, a.s, __int_as_float(a.arg), __int_as_float(a.bad));
}

__device__ __forceinline__ RowAcc load_partial(const RowPartial* p) {
  const float4 f = __ldcg(reinterpret_cast<const float4*>(p));
  return RowAcc{f.x, f.y, __float_as_int(f.z), __float_as_int(f.w)};
}

// Locate row `r` (0..rps-1) of sequence b: target rows 0..gamma, draft rows after.
template <bool kBf16>
__device__ __forceinline__ const char* row_ptr(const Pass1Params& p, int b, int r, bool& is_target) {
  constexpr size_t es = kBf16 ? 2 : 4;
  is_target = r <= p.gamma;
  if (is_target)
    return static_cast<const char*>(p.target) +
           (static_cast<size_t>(b) * (p.gamma + 1) + r) * static_cast<size_t>(p.V) * es;
  return static_cast<const char*>(p.draft) +
         (static_cast<size_t>(b) * p.gamma + (r - p.gamma - 1)) * static_cast<size_t>(p.V) * es;
}

// Publish a chunk partial and take the sequence's arrival ticket.  Returns
// true in every thread of the CTA that arrived last for sequence b.
template <int kThreads>
__device__ __forceinline__ bool publish_partial(const Pass1Params& p, int b, int r, int chunk,
                                                const RowAcc& a) {
  __shared__ int last;
  if (threadIdx.x == 0) {
    store_partial(p.part + (static_cast<size_t>(b) * p.rps + r) * p.nc + chunk, a);
    __threadfence();
    const unsigned t = atomicAdd(p.ticket + b, 1u);
    last = (t == static_cast<unsigned>(p.rps * p.nc - 1));
    if (last) p.ticket[b] = 0;  // leave the counter at zero for the next call
  }
  block_sync<kThreads>();
  if (last) __threadfence();
  return last;
}

// Stream one chunk from global memory (16-byte loads), reduce it, publish.
template <bool kBf16>
__device__ __forceinline__ bool pass1_chunk(const Pass1Params& p, int b, int r, int chunk) {
  __shared__ RowAcc scratch[kP1Threads / 32];
  bool is_target;
  const char* rp = row_ptr<kBf16>(p, b, r, is_target);
  const float T = __ldg(p.temps + b);
  const int mode = row_mode(T, is_target);
  RowAcc a{-INFINITY, 0.0f, 0x7fffffff, 0};
  if (mode == kRowLse) {
    const float c = __fdiv_rn(kLog2e, T);
    scan_chunk<kBf16, kRowLse, kP1Threads>(a, rp, p.V, chunk, p.nc, c);
    a = block_reduce_acc<kRowLse, kP1Threads>(a, c, scratch);
  } else if (mode == kRowArgmax) {
    scan_chunk<kBf16, kRowArgmax, kP1Threads>(a, rp, p.V, chunk, p.nc, 0.0f);
    a = block_reduce_acc<kRowArgmax, kP1Threads>(a, 0.0f, scratch);
  }
  return publish_partial<kP1Threads>(p, b, r, chunk, a);
}

// Combine the nc chunk partials of every row of sequence b into rows[].
// Called by all threads of the last-arriving CTA.
template <int kThreads>
__device__ __forceinline__ void combine_rows(const Pass1Params& p, int b, RowAcc* rows) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kThreads / 32;
  const float T = __ldg(p.temps + b);
  for (int r = warp; r < p.rps; r += kWarps) {
    const int mode = row_mode(T, r <= p.gamma);
    const float c = mode == kRowLse ? __fdiv_rn(kLog2e, T) : 0.0f;
    RowAcc a{-INFINITY, 0.0f, 0x7fffffff, 0};
    const RowPartial* pp = p.part + (static_cast<size_t>(b) * p.rps + r) * p.nc;
    for (int q = lane; q < p.nc; q += 32) {
      const RowAcc o = load_partial(pp + q);
      if (mode == kRowLse)
        acc_merge<kRowLse>(a, o, c);
      else
        acc_merge<kRowArgmax>(a, o, c);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      RowAcc o;
      o.m = __shfl_down_sync(0xffffffffu, a.m, off);
      o.s = __shfl_down_sync(0xffffffffu, a.s, off);
      o.arg = __shfl_down_sync(0xffffffffu, a.arg, off);
      o.bad = __shfl_down_sync(0xffffffffu, a.bad, off);
      if (mode == kRowLse)
        acc_merge<kRowLse>(a, o, c);
      else
        acc_merge<kRowArgmax>(a, o, c);
    }
    if (lane == 0) rows[r] = a;
  }
  block_sync<kThreads>();
}

}  // namespace sv
