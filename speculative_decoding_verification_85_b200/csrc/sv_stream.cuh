// sv_stream.cuh -- per-thread row reductions of the single-draft row kernel.
//
// A row-kernel CTA covers (sequence b, position i, vocabulary segment): target row i
// and draft row i over the same segment (position gamma: the target row
// alone).  The segment arrives in tiles of kTileVec 16-byte vectors per row;
// each thread copies its kTileRegs vectors of a tile into registers, then
// folds them into a running accumulator.
//
// Softmax sums use an integer reference exponent.  With c = log2(e) / T and
// R(m) = ceil(fl(m c)) for the running maximum m, a thread accumulates
//     S = sum_v 2^{z_v c - R(m)}
// where each exponent z_v c - R is one fused multiply-add (a single rounding;
// the largest term is at most 2^1).  Two partial sums with references R1 >= R2
// merge as S1 + S2 2^{R2 - R1}, a multiplication by an exact power of two.
// The row's sum relative to its maximum, s = sum_v 2^{(z_v - m) c}, is
// recovered once per row as S 2^{R(m) - m c} (in fp64).
//
// Per bf16 element: one bit operation to widen, half of a packed fp32x2 FMA,
// one MUFU ex2, half of a packed fp32x2 add; the tile maximum costs one
// packed bf16x2 max per two elements.
#pragma once

#include "sv_device.cuh"
#include "sv_internal.h"
#include "sv_rows.cuh"

namespace sv {

constexpr int kTileThreads = 256;                   // threads of a row-kernel CTA
constexpr int kTileRegs = 4;                        // vectors per thread per row per tile
constexpr int kTileVec = kTileThreads * kTileRegs;  // 16-byte vectors per row per tile (16 KB)

__device__ __forceinline__ uint32_t hmax2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Exact 2^d for an integral d <= 0 (0 below the normal range, and for NaN).
// The integer is read from the mantissa of d + 1.5 2^23 (no conversion unit).
__device__ __forceinline__ float exp2_int(float d) {
  if (!(d >= -126.0f)) return 0.0f;
  const int k = __float_as_int(d + 12582912.0f) - 0x4B400000;
  return __int_as_float((k + 127) << 23);
}

// Reference exponent R(m) = ceil(fl(m c)); the same operations everywhere.
__device__ __forceinline__ float ref_exp(float m, float c) { return ceilf(__fmul_rn(m, c)); }

// Running reduction of one row by one thread.
struct RunAcc {
  float m;   // running raw maximum (-inf: nothing yet)
  float R;   // R(m) (0 while m = -inf)
  float2 s;  // packed sum of 2^{z c - R} (softmax rows)
  int arg;   // first index of the maximum (greedy rows)
  int bad;   // saw NaN
  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    R = 0.0f;
    s = make_float2(0.0f, 0.0f);
    arg = 0x7fffffff;
    bad = 0;
  }
  // Greedy rows: {max, -, first index, bad}.
  __device__ __forceinline__ RowAcc argmax_row() const { return RowAcc{m, 0.0f, arg, bad}; }
  // Softmax rows: {max, S, R (in the index slot; -inf when empty), bad}.
  __device__ __forceinline__ RowAcc lse_row() const {
    return RowAcc{m, s.x + s.y, __float_as_int(m == -INFINITY ? -INFINITY : R), bad};
  }
};

// Move the running maximum up to tm (> m): new reference, rescale the sum.
__device__ __forceinline__ void lift_ref(RunAcc& a, float tm, float c) {
  const float Rn = ref_exp(tm, c);
  if (a.m != -INFINITY) {
    const float f = exp2_int(a.R - Rn);
    a.s = __fmul2_rn(a.s, make_float2(f, f));
  }
  a.m = tm;
  a.R = Rn;
}

template <bool kBf16>
struct Vec16;

template <>
struct Vec16<true> {  // 8 bf16
  static constexpr int kN = 8;
  static constexpr uint32_t kNegInf = 0xFF80FF80u;
  __device__ __forceinline__ static uint32_t pmax(const uint4& r) {
    return hmax2_nan(hmax2_nan(r.x, r.y), hmax2_nan(r.z, r.w));
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
  static constexpr uint32_t kNegInf = 0xFF800000u;
  __device__ __forceinline__ static float2 pair(const uint4& r, int k) {
    return k == 0 ? make_float2(__uint_as_float(r.x), __uint_as_float(r.y))
                  : make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
  }
  __device__ __forceinline__ static float at(const uint4& r, int e) {
    const uint32_t w = e == 0 ? r.x : (e == 1 ? r.y : (e == 2 ? r.z : r.w));
    return __uint_as_float(w);
  }
};

// Maximum of the thread's tile vectors (NaN if any element is NaN).
template <bool kBf16>
__device__ __forceinline__ float tile_max(const uint4 (&r)[kTileRegs]) {
  if constexpr (kBf16) {
    uint32_t m = Vec16<true>::pmax(r[0]);
#pragma unroll
    for (int j = 1; j < kTileRegs; ++j) m = hmax2_nan(m, Vec16<true>::pmax(r[j]));
    return max_nan(bf16_lo(m), bf16_hi(m));
  } else {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < kTileRegs; ++j)
      m = max_nan(max_nan(m, max_nan(__uint_as_float(r[j].x), __uint_as_float(r[j].y))),
                  max_nan(__uint_as_float(r[j].z), __uint_as_float(r[j].w)));
    return m;
  }
}

// Load the thread's vectors of the tile starting at vector kb; vectors at or
// beyond k1 read as -inf.
template <bool kBf16>
__device__ __forceinline__ void load_tile(const uint4* vp, int kb, int k1, uint4 (&r)[kTileRegs]) {
  constexpr uint32_t ninf = Vec16<kBf16>::kNegInf;
#pragma unroll
  for (int j = 0; j < kTileRegs; ++j) {
    const int k = kb + static_cast<int>(threadIdx.x) + j * kTileThreads;
    r[j] = k < k1 ? ld_stream(vp + k) : make_uint4(ninf, ninf, ninf, ninf);
  }
}

__device__ __forceinline__ float2 ex2_pair(float2 d) {
  return make_float2(ex2_approx(d.x), ex2_approx(d.y));
}

// Fold a tile into a softmax-sum accumulator.
template <bool kBf16>
__device__ __forceinline__ void lse_tile(RunAcc& a, const uint4 (&r)[kTileRegs], float c) {
  using V = Vec16<kBf16>;
  const float tm = tile_max<kBf16>(r);
  if (tm != tm) {
    a.bad = 1;
    return;
  }
  if (tm > a.m) lift_ref(a, tm, c);
  const float2 nr = make_float2(-a.R, -a.R), cc = make_float2(c, c);
  // one partial sum per vector, so the adds form kTileRegs independent chains
  float2 acc[kTileRegs];
#pragma unroll
  for (int j = 0; j < kTileRegs; ++j) {
    acc[j] = ex2_pair(__ffma2_rn(V::pair(r[j], 0), cc, nr));
#pragma unroll
    for (int k = 1; k < V::kN / 2; ++k)
      acc[j] = __fadd2_rn(acc[j], ex2_pair(__ffma2_rn(V::pair(r[j], k), cc, nr)));
  }
#pragma unroll
  for (int j = 1; j < kTileRegs; ++j) acc[0] = __fadd2_rn(acc[0], acc[j]);
  a.s = __fadd2_rn(a.s, acc[0]);
}

// Fold a tile into a first-argmax accumulator; v0 is the row index of the
// first element of the thread's vector j = 0, later vectors follow at
// kTileThreads vectors' distance (increasing indices).
template <bool kBf16>
__device__ __forceinline__ void argmax_tile(RunAcc& a, const uint4 (&r)[kTileRegs], int v0) {
  using V = Vec16<kBf16>;
  const float tm = tile_max<kBf16>(r);
  if (tm != tm) {
    a.bad = 1;
    return;
  }
  if (tm > a.m) {
    a.m = tm;
    int arg = 0x7fffffff;
#pragma unroll
    for (int j = kTileRegs - 1; j >= 0; --j)
#pragma unroll
      for (int e = V::kN - 1; e >= 0; --e)
        if (V::at(r[j], e) == tm) arg = v0 + j * kTileThreads * V::kN + e;
    a.arg = arg;
  }
}

__device__ __forceinline__ void lse_scalar(RunAcc& a, float z, float c) {
  if (z != z) {
    a.bad = 1;
    return;
  }
  if (z > a.m) lift_ref(a, z, c);
  a.s.x += ex2_approx(fmaf(z, c, -a.R));
}

__device__ __forceinline__ void argmax_scalar(RunAcc& a, float z, int v) {
  if (z != z) {
    a.bad = 1;
    return;
  }
  // the head elements are visited after the body: keep the lowest index on ties
  if (z > a.m || (z == a.m && v < a.arg)) {
    a.m = z;
    a.arg = v;
  }
}

// Merge partial b into a.  Softmax rows ({m, S, R, bad}, R in the index
// slot): the larger maximum, and the sums brought to the larger reference
// by an exact power of two; greedy rows: the larger maximum wins, ties keep
// the lower index.
__device__ __forceinline__ void merge_ref(RowAcc& a, const RowAcc& b, bool argmax) {
  a.bad |= b.bad;
  if (argmax) {
    if (b.m > a.m || (b.m == a.m && b.arg < a.arg)) {
      a.m = b.m;
      a.arg = b.arg;
    }
    return;
  }
  a.m = fmaxf(a.m, b.m);
  const float Ra = __int_as_float(a.arg), Rb = __int_as_float(b.arg);
  if (Rb > Ra) {
    a.s = b.s + a.s * exp2_int(Ra - Rb);
    a.arg = b.arg;
  } else {
    a.s += b.s * exp2_int(Rb - Ra);
  }
}

__device__ __forceinline__ RowAcc shfl_xor_acc(const RowAcc& a, int off) {
  RowAcc o;
  o.m = __shfl_xor_sync(0xffffffffu, a.m, off);
  o.s = __shfl_xor_sync(0xffffffffu, a.s, off);
  o.arg = __shfl_xor_sync(0xffffffffu, a.arg, off);
  o.bad = __shfl_xor_sync(0xffffffffu, a.bad, off);
  return o;
}

// Butterfly merge over groups of `width` lanes (every lane ends with its
// group's result).
template <int width>
__device__ __forceinline__ void group_merge(RowAcc& a, bool argmax) {
#pragma unroll
  for (int off = width / 2; off > 0; off >>= 1) merge_ref(a, shfl_xor_acc(a, off), argmax);
}
__device__ __forceinline__ void warp_merge(RowAcc& a, bool argmax) { group_merge<32>(a, argmax); }

// Geometry of one row: unaligned head elements, then 16-byte body vectors,
// then the tail.
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
  __device__ __forceinline__ const uint4* body(const char* rp) const {
    return reinterpret_cast<const uint4*>(rp + static_cast<size_t>(head) * (kBf16 ? 2 : 4));
  }
};

}  // namespace sv
