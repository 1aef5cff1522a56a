// sv_cluster.cuh -- exchanges between the CTAs of a thread-block cluster.
#pragma once

#include "sv_device.cuh"

namespace sv {

// Distributed-shared-memory stores that complete a transaction on the
// destination CTA's mbarrier: the receiver waits on its own barrier, with no
// cluster-wide barrier per exchange.
__device__ __forceinline__ uint32_t mapa(const void* p, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_async_f64(uint32_t addr, double v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];"
               ::"r"(addr), "l"(__double_as_longlong(v)), "r"(bar) : "memory");
}
__device__ __forceinline__ void st_async_f4(uint32_t addr, float4 v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
               ::"r"(addr), "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)),
               "r"(__float_as_uint(v.z)), "r"(__float_as_uint(v.w)), "r"(bar)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (kWaitLimitNs) for a phase of an exchange barrier.
__device__ __forceinline__ bool xbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int k = 0; k < 64; ++k)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}


// Stage the slice [v0, v0 + n) of nq rows (row q starts at grow(q) in global
// memory) into shared memory: row q's slice goes to srows + q rowstride +
// (its global address mod 16), so the aligned body of each row slice is one
// bulk copy, completing on its own barrier bars[q] (initialised, phase 0,
// and ordered before this call by a CTA barrier); issued without waiting:
// thread q issues row q's bulk copy and all kThreads threads copy the
// unaligned heads and tails.  Returns
// whether there were any (the same answer in every thread); if so, a CTA
// barrier must order those scalar copies before use.  A thread may use row q
// once mbar_wait(&bars[q], 0) returns true, so a row is processed while
// later rows are still in flight.
template <size_t es, int kThreads, typename RowFn>
__device__ __forceinline__ bool stage_rows_issue(RowFn grow, int nq, int v0, int n, char* srows,
                                                 int rowstride, uint64_t* bars) {
  const int tid = threadIdx.x;
  auto geom = [&](int q, const char*& g, uint32_t& hb, uint32_t& body, char*& sdst) {
    g = grow(q) + static_cast<size_t>(v0) * es;
    const uintptr_t ga = reinterpret_cast<uintptr_t>(g);
    hb = min(static_cast<uint32_t>((16u - (ga & 15u)) & 15u), static_cast<uint32_t>(n * es));
    body = (static_cast<uint32_t>(n * es) - hb) / 16u * 16u;
    sdst = srows + static_cast<size_t>(q) * rowstride + (ga & 15u);
  };
  // the bulk copies, thread q issuing row q's (one instruction per warp)
  for (int q = tid; q < nq; q += kThreads) {
    const char* g;
    uint32_t hb, body;
    char* sdst;
    geom(q, g, hb, body, sdst);
    if (body) {
      mbar_arrive_expect_tx(&bars[q], body);
      bulk_g2s(sdst + hb, g + hb, body, &bars[q]);
    } else {
      mbar_arrive(&bars[q]);
    }
  }
  // the unaligned heads and tails, by all threads
  bool scalar = false;  // some row slice has an unaligned head or tail
  for (int q = 0; q < nq; ++q) {
    const char* g;
    uint32_t hb, body;
    char* sdst;
    geom(q, g, hb, body, sdst);
    const int h = static_cast<int>(hb / es), t0 = static_cast<int>((hb + body) / es);
    if (h == 0 && t0 >= n) continue;
    scalar = true;
    for (int e = tid; e < h; e += kThreads) memcpy(sdst + e * es, g + e * es, es);
    for (int e = t0 + tid; e < n; e += kThreads) memcpy(sdst + e * es, g + e * es, es);
  }
  return scalar;
}

}  // namespace sv
