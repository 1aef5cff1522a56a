// sv_device.cuh -- device-side building blocks of the verifier (sm_100a).
//
// Philox4x32-10 here is an independent implementation of Salmon, Moraes,
// Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): each of
// the 10 rounds multiplies counter words 0 and 2 by fixed odd constants,
// xors the high halves into words 1 and 3 together with the round key, and
// the key is advanced by the Weyl increments between rounds.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sv {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWarp = 32;

// Counter tags (4th counter word = tag << 24 | k << 12 | pos).
constexpr uint32_t kTagAccept = 1;
constexpr uint32_t kTagGumbel = 2;
constexpr uint32_t kTagMdEta = 3;
constexpr uint32_t kTagMdGumbel = 4;
constexpr uint32_t kTagGroup = 7;   // group-level noise of the single-draft draw
constexpr int kRaceGroup = 1024;    // vocabulary entries per group of the single-draft draw

// Pass-2 modes of a sequence.
constexpr int kModeNone = 0;      // nothing to draw (greedy or invalid)
constexpr int kModeResidual = 1;  // draw from max(p_j - q_j, 0)
constexpr int kModeBonus = 2;     // draw from p_gamma

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    // one wide multiply gives both halves of each 32 x 32 -> 64-bit product
    const uint64_t p0 = static_cast<uint64_t>(c.x) * 0xD2511F53u;
    const uint64_t p1 = static_cast<uint64_t>(c.z) * 0xCD9E8D57u;
    const uint32_t lo0 = static_cast<uint32_t>(p0), hi0 = static_cast<uint32_t>(p0 >> 32);
    const uint32_t lo1 = static_cast<uint32_t>(p1), hi1 = static_cast<uint32_t>(p1 >> 32);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Keyed stream: key (lo32(seed), hi32(seed)); counter (c0, b, lo32(step), tag|k|pos).
__device__ __forceinline__ uint4 keyed_block(uint64_t seed, uint32_t step, uint32_t tag,
                                             uint32_t b, uint32_t k, uint32_t pos,
                                             uint32_t c0) {
  return philox4x32_10(make_uint4(c0, b, step, (tag << 24) | (k << 12) | pos),
                       static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
}

// The same stream with the key schedule and the fixed counter words worked
// out once, for many blocks that differ only in c0 (one draw race).
struct PhiloxStream {
  uint32_t k0[10], k1[10];  // round keys
  uint32_t c1, c2, c3;      // counter words 1..3
  __device__ __forceinline__ PhiloxStream(uint64_t seed, uint32_t step, uint32_t tag, uint32_t b,
                                          uint32_t k, uint32_t pos) {
    uint32_t a = static_cast<uint32_t>(seed), d = static_cast<uint32_t>(seed >> 32);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      k0[r] = a;
      k1[r] = d;
      a += 0x9E3779B9u;
      d += 0xBB67AE85u;
    }
    c1 = b;
    c2 = step;
    c3 = (tag << 24) | (k << 12) | pos;
  }
  __device__ __forceinline__ uint4 block(uint32_t c0) const {
    uint4 c = make_uint4(c0, c1, c2, c3);
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      const uint64_t p0 = static_cast<uint64_t>(c.x) * 0xD2511F53u;
      const uint64_t p1 = static_cast<uint64_t>(c.z) * 0xCD9E8D57u;
      c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k0[r], static_cast<uint32_t>(p1),
                     static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k1[r], static_cast<uint32_t>(p0));
    }
    return c;
  }
};

__device__ __forceinline__ uint32_t word_of(const uint4& r, int w) {
  return w == 0 ? r.x : (w == 1 ? r.y : (w == 2 ? r.z : r.w));
}

// Acceptance uniform in [0, 1): (x >> 8) * 2^-24 (exact in fp32 and fp64).
__device__ __forceinline__ double accept_uniform(uint32_t x) {
  return static_cast<double>(x >> 8) * 0x1p-24;
}

// For the Gumbel uniform U = (2 (x >> 9) + 1) * 2^-24, return t = 1 - U,
// which is again an odd multiple of 2^-24 and exact in fp32: the mantissa
// trick builds 1 + n' 2^-23 with n' = ~x >> 9 and subtracts 1 - 2^-24.
__device__ __forceinline__ float gumbel_one_minus_u(uint32_t x) {
  return __uint_as_float(0x3F800000u | ((~x) >> 9)) - 0x1.fffffep-1f;
}

// E = -ln U evaluated as -log1p(-(1 - U)), accurate for U close to 1 (where
// E is small and the draw is most likely to win).  The race winner
// argmax_v w_v / E_v equals the Gumbel-max argmax_v (ln w_v - ln E_v).
__device__ __forceinline__ float exponential_from_bits(uint32_t x) {
  return -log1pf(-gumbel_one_minus_u(x));
}

// Raw MUFU base-2 exponential (flush-to-zero; relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// NaN-propagating maximum.
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Arrival ticket with acquire-release semantics: releases this thread's
// earlier stores and, for the last arriver, acquires everything the earlier
// arrivers released (a CTA barrier then extends that to the whole CTA).
__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* p) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}
// 16-byte load of data read once (no L1 allocation).
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_at(const uint16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(p + i)) << 16);
}

template <bool kBf16>
__device__ __forceinline__ float logit_at(const void* row, int64_t v) {
  if constexpr (kBf16) {
    return bf16_at(static_cast<const uint16_t*>(row), v);
  } else {
    return __ldg(static_cast<const float*>(row) + v);
  }
}

// Combine two (max, scaled sum) pairs of a base-2 log-sum-exp with scale c:
// s_i = sum 2^{(z - m_i) c}.  Pairs with m = -inf carry nothing.
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2, float c) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  if (m2 > m) {
    s = s * ex2_approx((m - m2) * c) + s2;
    m = m2;
  } else {
    s = s + s2 * ex2_approx((m2 - m) * c);
  }
}

// (max, first index) pair: larger value wins; equal values keep the lower index.
__device__ __forceinline__ void argmax_merge(float& m, int& a, float m2, int a2) {
  if (m2 > m || (m2 == m && a2 < a)) {
    m = m2;
    a = a2;
  }
}

// Barrier among the first kThreads threads of the block (named barrier 1).
// Kernels whose CTA has extra warps (a producer warp) use it for the threads
// that do the reductions; with kThreads == blockDim.x it is a block barrier.
template <int kThreads>
__device__ __forceinline__ void block_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}

// Exponential-race candidate (w, E, index): w / E larger wins, ties go to
// the lower index; w == 0 means "no candidate".
__device__ __forceinline__ bool race_better(float w, float e, int idx, float bw, float be,
                                            int bidx) {
  if (!(w > 0.0f)) return false;
  if (!(bw > 0.0f)) return true;
  const float lhs = w * be, rhs = bw * e;
  return lhs > rhs || (lhs == rhs && idx < bidx);
}


// ------------------------------------------------ async copies and flags
// Bulk prefetch of [p, p + bytes) into L2 (p and bytes multiples of 16); no
// destination, no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Shared-memory address of a generic pointer to this CTA's shared memory.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Arrive and add `bytes` to the transaction count the current phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Nanoseconds of the GPU's global timer.
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait on another thread's progress gives up after this long and
// reports it (no correct run comes anywhere near it).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Wait for the phase of parity `parity` to complete; false when the wait
// ran out of time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int k = 0; k < 64; ++k)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing
// `bytes` of the barrier's transaction count.  dst, src 16-byte aligned;
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(smem_addr(p)));
  return r;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

}  // namespace sv

namespace sv {

// Block-wide reduction of exponential-race candidates.  The winner is
// returned to EVERY thread of the block (so a branch on it is uniform and may
// contain barriers).  `scratch` holds kThreads / 32 float4 slots.
template <int kThreads>
__device__ __forceinline__ void race_reduce(float& bw, float& be, int& bi, float4* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float w2 = __shfl_down_sync(0xffffffffu, bw, off);
    const float e2 = __shfl_down_sync(0xffffffffu, be, off);
    const int i2 = __shfl_down_sync(0xffffffffu, bi, off);
    if (race_better(w2, e2, i2, bw, be, bi)) {
      bw = w2;
      be = e2;
      bi = i2;
    }
  }
  if (lane == 0) scratch[warp] = make_float4(bw, be, __int_as_float(bi), 0.0f);
  block_sync<kThreads>();
  if (warp == 0) {
    constexpr int kWarps = kThreads / 32;
    const float4 q = lane < kWarps ? scratch[lane] : make_float4(0.0f, 1.0f, __int_as_float(0x7fffffff), 0.0f);
    bw = q.x;
    be = q.y;
    bi = __float_as_int(q.z);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float w2 = __shfl_down_sync(0xffffffffu, bw, off);
      const float e2 = __shfl_down_sync(0xffffffffu, be, off);
      const int i2 = __shfl_down_sync(0xffffffffu, bi, off);
      if (race_better(w2, e2, i2, bw, be, bi)) {
        bw = w2;
        be = e2;
        bi = i2;
      }
    }
    if (lane == 0) scratch[0] = make_float4(bw, be, __int_as_float(bi), 0.0f);
  }
  block_sync<kThreads>();
  const float4 r = scratch[0];
  bw = r.x;
  be = r.y;
  bi = __float_as_int(r.z);
  block_sync<kThreads>();  // scratch may be reused right after
}

// Block-wide fp64 sum, result returned to every thread.  `red` holds 33
// doubles.  Contains __syncthreads().
template <int kThreads>
__device__ __forceinline__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  if (lane == 0) red[warp] = v;
  block_sync<kThreads>();
  if (warp == 0) {
    constexpr int kWarps = kThreads / 32;
    v = lane < kWarps ? red[lane] : 0.0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    if (lane == 0) red[32] = v;
  }
  block_sync<kThreads>();
  return red[32];
}

}  // namespace sv
