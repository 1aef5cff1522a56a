// sv_noalloc.cu -- spec_verify without a caller-provided workspace.
//
// Some callers cannot allocate device memory when they verify: an inference
// engine that reserves nearly all of the GPU's memory up front for weights
// and KV cache, or a runtime whose decode path must never enter an
// allocator.  For them spec_verify_noalloc runs the same kernels as
// spec_verify with scratch memory taken from a fixed array in the library's
// own device memory (it exists from the moment the library's module is
// loaded), so the call itself allocates nothing.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "spec_verify.h"
#include "sv_internal.h"

namespace sv {
namespace {

// The workspace of spec_verify_noalloc: one per device the module is loaded on.
__device__ __align__(256) unsigned char g_noalloc_ws[SV_NOALLOC_MAX_WORKSPACE];

struct NoAllocState {
  void* ptr = nullptr;  // device address of g_noalloc_ws on this device
  bool ready = false;
};

// Per device: the array's address (cudaGetSymbolAddress, with that device
// current) and a one-time clear of its counter header on the first call's
// stream.  Returns SV_OK or an error status.
int noalloc_workspace(void** out, cudaStream_t stream) {
  static std::mutex mu;
  static NoAllocState state[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return set_error(SV_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(mu);
  NoAllocState& s = state[dev];
  if (!s.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess)
      return set_error(SV_ERR_CUDA, "cudaGetSymbolAddress (no-alloc workspace): %s",
                       cudaGetErrorString(e));
    // The arrival counters must start at zero; every call leaves them so.
    e = cudaMemsetAsync(p, 0, kHeaderBytes, stream);
    if (e != cudaSuccess)
      return set_error(SV_ERR_CUDA, "cudaMemsetAsync (no-alloc workspace): %s", cudaGetErrorString(e));
    s.ptr = p;
    s.ready = true;
  }
  *out = s.ptr;
  return SV_OK;
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" size_t spec_verify_noalloc_max_workspace(void) { return SV_NOALLOC_MAX_WORKSPACE; }

extern "C" int spec_verify_noalloc(const void* target_logits, const void* draft_logits,
                                   const int32_t* draft_tokens, const float* temps, int B,
                                   int gamma, int V, int dtype, uint64_t seed, uint64_t step,
                                   int32_t* out_accept_len, int32_t* out_tokens,
                                   float* out_target_logp, float* out_draft_logp, void* stream) {
  const size_t need = spec_verify_workspace_size(B, gamma, V, dtype);
  if (B > 0 && need == 0)  // a bad shape: spec_verify reports it before any CUDA work
    return spec_verify(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, seed,
                       step, out_accept_len, out_tokens, out_target_logp, out_draft_logp, nullptr,
                       0, stream);
  if (B > 0 && need > SV_NOALLOC_MAX_WORKSPACE)
    return set_error(SV_ERR_WORKSPACE,
                     "spec_verify_noalloc: this shape needs %zu bytes of workspace, more than "
                     "the fixed %zu (use spec_verify with a caller workspace)",
                     need, static_cast<size_t>(SV_NOALLOC_MAX_WORKSPACE));
  void* ws = nullptr;
  if (B > 0) {
    const int rc = noalloc_workspace(&ws, static_cast<cudaStream_t>(stream));
    if (rc != SV_OK) return rc;
  }
  return spec_verify(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, seed,
                     step, out_accept_len, out_tokens, out_target_logp, out_draft_logp, ws,
                     SV_NOALLOC_MAX_WORKSPACE, stream);
}
