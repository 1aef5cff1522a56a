// sv_stream.cuh -- row-pair streaming reduction for the fused single-draft
// kernel.
//
// A pass-1 work item is (sequence b, position i, vocabulary segment): target
// row i and draft row i over the same segment (position gamma: the target row
// alone).  The producer warp stages the item in pieces of up to kStageVec
// 16-byte vectors per row; the consumer threads keep running per-row
// accumulators in registers across the pieces and publish one partial per item.
//
// Arithmetic per bf16 element: exact widening, NaN-propagating max on packed
// bf16x2, then (z - max) * log2(e)/T with packed fp32x2 add/mul, one MUFU
// ex2, and a packed fp32x2 running sum.
#pragma once

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace sv {

constexpr int kStageVec = 1024;  // 16-byte vectors per row per stage (16 KB)

__device__ __forceinline__ uint32_t hmax2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Per-thread running reduction of one row.
struct RunAcc {
  float m;    // running raw max
  float2 s;   // packed sum of 2^{(z - m) c}
  int arg;    // first index of the max (greedy rows)
  int bad;    // saw NaN
  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    s = make_float2(0.0f, 0.0f);
    arg = 0x7fffffff;
    bad = 0;
  }
  __device__ __forceinline__ RowAcc row() const { return RowAcc{m, s.x + s.y, arg, bad}; }
};

// Move the running max to vm (> m), rescaling the sum.
__device__ __forceinline__ void lift_max(RunAcc& a, float vm, float c) {
  if (a.m != -INFINITY) {
    const float f = ex2_approx((a.m - vm) * c);
    a.s = __fmul2_rn(a.s, make_float2(f, f));
  }
  a.m = vm;
}

// 2^{(z - m) c} for a pair of logits.
__device__ __forceinline__ float2 exp_pair(float2 z, float2 nm, float2 cc) {
  const float2 d = __fmul2_rn(__fadd2_rn(z, nm), cc);
  return make_float2(ex2_approx(d.x), ex2_approx(d.y));
}

template <bool kBf16>
struct Vec16;

template <>
struct Vec16<true> {  // 8 bf16
  static constexpr int kN = 8;
  __device__ __forceinline__ static float vmax(const uint4& r) {
    const uint32_t mm = hmax2_nan(hmax2_nan(r.x, r.y), hmax2_nan(r.z, r.w));
    return max_nan(bf16_lo(mm), bf16_hi(mm));
  }
  __device__ __forceinline__ static float2 pair(const uint4& r, int k) {
    const uint32_t w = k == 0 ? r.x : (k == 1 ? r.y : (k == 2 ? r.z : r.w));
    return make_float2(bf16_lo(w), bf16_hi(w));
  }
  __device__ __forceinline__ static float at(const uint4& r, int e) {
    const float2 p = pair(r, e >> 1);
    return (e & 1) ? p.y : p.x;
  }
};

template <>
struct Vec16<false> {  // 4 fp32
  static constexpr int kN = 4;
  __device__ __forceinline__ static float vmax(const uint4& r) {
    return max_nan(max_nan(__uint_as_float(r.x), __uint_as_float(r.y)),
                   max_nan(__uint_as_float(r.z), __uint_as_float(r.w)));
  }
  __device__ __forceinline__ static float2 pair(const uint4& r, int k) {
    return k == 0 ? make_float2(__uint_as_float(r.x), __uint_as_float(r.y))
                  : make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
  }
  __device__ __forceinline__ static float at(const uint4& r, int e) {
    const uint32_t w = e == 0 ? r.x : (e == 1 ? r.y : (e == 2 ? r.z : r.w));
    return __uint_as_float(w);
  }
};

template <bool kBf16>
__device__ __forceinline__ void lse_vec(RunAcc& a, const uint4& r, float c) {
  using V = Vec16<kBf16>;
  const float vm = V::vmax(r);
  if (vm != vm) {
    a.bad = 1;
    return;
  }
  if (vm == -INFINITY) return;
  if (vm > a.m) lift_max(a, vm, c);
  const float2 nm = make_float2(-a.m, -a.m), cc = make_float2(c, c);
  if constexpr (kBf16) {
    const float2 e0 = exp_pair(V::pair(r, 0), nm, cc);
    const float2 e1 = exp_pair(V::pair(r, 1), nm, cc);
    const float2 e2 = exp_pair(V::pair(r, 2), nm, cc);
    const float2 e3 = exp_pair(V::pair(r, 3), nm, cc);
    a.s = __fadd2_rn(a.s, __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3)));
  } else {
    const float2 e0 = exp_pair(V::pair(r, 0), nm, cc);
    const float2 e1 = exp_pair(V::pair(r, 1), nm, cc);
    a.s = __fadd2_rn(a.s, __fadd2_rn(e0, e1));
  }
}

template <bool kBf16>
__device__ __forceinline__ void argmax_vec(RunAcc& a, const uint4& r, int v0) {
  using V = Vec16<kBf16>;
  const float vm = V::vmax(r);
  if (vm != vm) {
    a.bad = 1;
    return;
  }
  if (vm > a.m) {
    a.m = vm;
#pragma unroll
    for (int e = V::kN - 1; e >= 0; --e)
      if (V::at(r, e) == vm) a.arg = v0 + e;
  }
}

// Sum of 2^{(z - m) c} over the elements of one vector (m fixed, finite).
template <bool kBf16>
__device__ __forceinline__ float2 exp_vec(const uint4& r, float2 nm, float2 cc) {
  using V = Vec16<kBf16>;
  if constexpr (kBf16) {
    const float2 e0 = exp_pair(V::pair(r, 0), nm, cc);
    const float2 e1 = exp_pair(V::pair(r, 1), nm, cc);
    const float2 e2 = exp_pair(V::pair(r, 2), nm, cc);
    const float2 e3 = exp_pair(V::pair(r, 3), nm, cc);
    return __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3));
  } else {
    return __fadd2_rn(exp_pair(V::pair(r, 0), nm, cc), exp_pair(V::pair(r, 1), nm, cc));
  }
}

// Fold kR vectors of one thread (r[j] valid for j < n) into the running
// accumulator: one max over all of them first, at most one rescale, then
// independent exponentials (instruction-level parallelism across vectors).
template <bool kBf16, int kR>
__device__ __forceinline__ void lse_block(RunAcc& a, const uint4 (&r)[kR], int n, float c) {
  using V = Vec16<kBf16>;
  float vm = -INFINITY, mj[kR];
  bool nan = false;
#pragma unroll
  for (int j = 0; j < kR; ++j) {
    mj[j] = -INFINITY;
    if (j < n) {
      mj[j] = V::vmax(r[j]);
      nan |= (mj[j] != mj[j]);
      vm = fmaxf(vm, mj[j]);
    }
  }
  if (nan) {
    a.bad = 1;
    return;
  }
  if (vm == -INFINITY) return;
  if (vm > a.m) lift_max(a, vm, c);
  const float2 nm = make_float2(-a.m, -a.m), cc = make_float2(c, c);
  float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < kR; ++j)
    // a vector whose largest term is below 2^-126 contributes only flushed
    // zeros: skip its exponentials (same result)
    if (j < n && (mj[j] - a.m) * c >= -126.0f) acc = __fadd2_rn(acc, exp_vec<kBf16>(r[j], nm, cc));
  a.s = __fadd2_rn(a.s, acc);
}

template <bool kBf16, int kR>
__device__ __forceinline__ void argmax_block(RunAcc& a, const uint4 (&r)[kR], int n, const int (&v0)[kR]) {
#pragma unroll
  for (int j = 0; j < kR; ++j)
    if (j < n) argmax_vec<kBf16>(a, r[j], v0[j]);
}

__device__ __forceinline__ void lse_scalar(RunAcc& a, float z, float c) {
  if (z != z) {
    a.bad = 1;
    return;
  }
  if (z == -INFINITY) return;
  if (z > a.m) lift_max(a, z, c);
  a.s.x += ex2_approx((z - a.m) * c);
}

__device__ __forceinline__ void argmax_scalar(RunAcc& a, float z, int v) {
  if (z != z) {
    a.bad = 1;
    return;
  }
  if (z > a.m) {
    a.m = z;
    a.arg = v;
  }
}

// Geometry of one row: unaligned head elements, 16-byte body vectors, tail;
// the body is split into nseg segments, each staged in pieces of kStageVec.
template <bool kBf16>
struct RowGeom {
  int head, nvec, tail0;
  __device__ __forceinline__ RowGeom(const char* rp, int V) {
    constexpr int es = kBf16 ? 2 : 4;
    const uintptr_t addr = reinterpret_cast<uintptr_t>(rp);
    head = static_cast<int>(((16u - (addr & 15u)) & 15u) / es);
    if (head > V) head = V;
    nvec = (V - head) / Vec16<kBf16>::kN;
    tail0 = head + nvec * Vec16<kBf16>::kN;
  }
  // Vectors [k0, k1) of segment `seg` of `nseg`.
  __device__ __forceinline__ void segment(int seg, int nseg, int& k0, int& k1) const {
    const int cs = (nvec + nseg - 1) / nseg;
    k0 = min(nvec, seg * cs);
    k1 = min(nvec, k0 + cs);
  }
  __device__ __forceinline__ int stages(int seg, int nseg) const {
    int k0, k1;
    segment(seg, nseg, k0, k1);
    return (k1 - k0 + kStageVec - 1) / kStageVec;
  }
  __device__ __forceinline__ const char* vec_ptr(const char* rp, int k) const {
    return rp + static_cast<size_t>(head) * (kBf16 ? 2 : 4) + static_cast<size_t>(k) * 16;
  }
};

}  // namespace sv
