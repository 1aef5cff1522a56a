// sv_rows.cuh -- per-row statistics shared by the verification kernels.
//
// Per row the kernels need what the acceptance test and the correction draw
// use: the raw maximum (NaN-propagating), the base-2 scaled sum
// S = sum_v 2^{(z_v - max) log2(e) / T} (the softmax normaliser of z / T), and,
// for greedy rows, the first index of the maximum.
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

template <int kMode>
__device__ __forceinline__ void acc_merge(RowAcc& a, const RowAcc& o, float c) {
  a.bad |= o.bad;
  if constexpr (kMode == kRowLse) {
    lse_merge(a.m, a.s, o.m, o.s, c);
  } else {
    argmax_merge(a.m, a.arg, o.m, o.arg);
  }
}

}  // namespace sv
