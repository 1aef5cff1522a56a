// sv_api.cu -- the C ABI: argument checks, workspace layout, host-buffer path.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "spec_verify.h"
#include "spec_verify_shard.h"
#include "sv_internal.h"

namespace sv {

namespace {
thread_local char g_err[512] = "no error";

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool sizes_ok(int B, int g, int V, int dtype) {
  return B >= 0 && B <= SV_MAX_BATCH && g >= 1 && g <= SV_MAX_GAMMA && V >= 1 && (dtype == SV_F32 || dtype == SV_BF16);
}
}  // namespace

int set_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return status;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return set_error(SV_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return SV_OK;
}

// Accept only compute capability 10.0 (the binary holds sm_100a code only).
int check_device() {
  static std::mutex mu;
  static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64) {
    std::lock_guard<std::mutex> lk(mu);
    if (cached[dev] == 0) {
      int major = 0, minor = 0;
      e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
      if (e != cudaSuccess)
        return set_error(SV_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
      cached[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    if (cached[dev] == 2)
      return set_error(SV_ERR_UNSUPPORTED, "device %d is not sm_100 (this library is built for sm_100a)", dev);
  }
  return SV_OK;
}

Layout layout_single(int B, int gamma, int V, int dtype) {
  Layout l{};
  l.nc = row_segments(V, dtype);
  l.nc2 = draw_chunks(V);
  l.ticket1 = 0;
  l.ticket2 = kSeqSlots;
  l.ready = 2 * kSeqSlots;
  size_t off = kHeaderBytes;
  l.part1 = off;  // row-pair partials: [B][gamma + 1][nseg] x 2 x 16 bytes
  off += up(static_cast<size_t>(B) * (gamma + 1) * l.nc * 2 * sizeof(float4));
  l.info = off;
  off += up(static_cast<size_t>(B) * sizeof(SeqInfo));
  l.part2 = off;
  off += up(static_cast<size_t>(B) * l.nc2 * sizeof(RacePartial));
  l.resid = off;  // the draft tokens' gathered logits: [B][gamma][nseg][2] fp32
  off += up(static_cast<size_t>(B) * gamma * l.nc * 2 * sizeof(float));
  l.total = off;
  return l;
}

Layout layout_multi(int B, int K, int L, int V, int dtype) {
  (void)K;
  (void)L;
  (void)dtype;
  Layout l{};
  l.nc = 0;
  l.nc2 = 0;
  l.ticket1 = 0;
  l.ticket2 = kSeqSlots;
  l.ready = 2 * kSeqSlots;
  size_t off = kHeaderBytes;
  l.resid = off;  // residual laws R (two per sequence) when they do not fit on chip
  off += up(multidraft_global_bytes(B, V));
  l.part1 = l.info = l.part2 = 0;
  l.total = off;
  return l;
}

}  // namespace sv

using namespace sv;

extern "C" {

int spec_verify_version(void) { return (1 << 16) | 1; }

const char* spec_verify_last_error(void) { return g_err; }

size_t spec_verify_workspace_size(int B, int gamma, int V, int dtype) {
  if (!sizes_ok(B, gamma, V, dtype)) return 0;
  return layout_single(B, gamma, V, dtype).total;
}

size_t spec_verify_multidraft_workspace_size(int B, int K, int L, int V, int dtype) {
  if (!sizes_ok(B, L, V, dtype) || K < 1 || K > SV_MAX_DRAFTS) return 0;
  return layout_multi(B, K, L, V, dtype).total;
}

int spec_verify_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace && workspace_bytes) return set_error(SV_ERR_WORKSPACE, "workspace is NULL");
  if (!workspace_bytes) return SV_OK;
  const cudaError_t e =
      cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  return SV_OK;
}

static int check_common(const void* t, const void* d, const void* x, const void* temps, int B,
                        int g, int V, int dtype, uint64_t step, const void* acc, const void* tok,
                        void* ws, size_t ws_bytes, size_t need) {
  if (dtype != SV_F32 && dtype != SV_BF16) return set_error(SV_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (B < 0 || B > SV_MAX_BATCH)
    return set_error(SV_ERR_INVALID_ARG, "B must be in [0, %d] (got %d)", SV_MAX_BATCH, B);
  if (g < 1 || g > SV_MAX_GAMMA)
    return set_error(SV_ERR_INVALID_ARG, "draft length must be in [1, %d] (got %d)", SV_MAX_GAMMA, g);
  if (V < 1) return set_error(SV_ERR_INVALID_ARG, "V must be >= 1 (got %d)", V);
  if (step >> 32) return set_error(SV_ERR_INVALID_ARG, "step must be < 2^32");
  if (B == 0) return SV_OK;
  if (!t || !d || !x || !temps || !acc || !tok)
    return set_error(SV_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!ws) return set_error(SV_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256)
    return set_error(SV_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return set_error(SV_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  const size_t es = dtype == SV_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(t) % es || reinterpret_cast<uintptr_t>(d) % es ||
      reinterpret_cast<uintptr_t>(x) % 4 || reinterpret_cast<uintptr_t>(temps) % 4)
    return set_error(SV_ERR_INVALID_ARG, "input pointers must be aligned to their element size");
  return SV_OK;
}

int spec_verify(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
                const float* temps, int B, int gamma, int V, int dtype, uint64_t seed,
                uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                float* out_target_logp, float* out_draft_logp, void* workspace,
                size_t workspace_bytes, void* stream) {
  const bool shape_ok = B > 0 && sizes_ok(B, gamma, V, dtype);
  const Layout lay = shape_ok ? layout_single(B, gamma, V, dtype) : Layout{};
  int rc = check_common(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, step,
                        out_accept_len, out_tokens, workspace, workspace_bytes, lay.total);
  if (rc != SV_OK || B == 0) return rc;
  if ((rc = check_device()) != SV_OK) return rc;
  return launch_single(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, seed,
                       step, out_accept_len, out_tokens, out_target_logp, out_draft_logp, workspace,
                       lay, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------- vocabulary shards
size_t spec_verify_shard_stats_bytes(int B, int gamma) {
  if (B < 0 || B > SV_MAX_BATCH || gamma < 1 || gamma > SV_MAX_GAMMA) return 0;
  return static_cast<size_t>(B) * (gamma + 1) * 3 * sizeof(float4);
}

size_t spec_verify_shard_candidate_bytes(int B) {
  if (B < 0 || B > SV_MAX_BATCH) return 0;
  return static_cast<size_t>(B) * sizeof(ShardCand);
}

static int check_shard(int V, int v0, int Vs) {
  if (v0 < 0 || Vs < 1 || static_cast<long long>(v0) + Vs > V)
    return set_error(SV_ERR_INVALID_ARG, "shard [v0, v0 + Vs) = [%d, %lld) must lie in [0, V = %d)",
                     v0, static_cast<long long>(v0) + Vs, V);
  if (v0 % SV_SHARD_ALIGN)
    return set_error(SV_ERR_INVALID_ARG, "shard offset v0 = %d must be a multiple of %d", v0,
                     SV_SHARD_ALIGN);
  if (v0 + Vs != V && Vs % SV_SHARD_ALIGN)
    return set_error(SV_ERR_INVALID_ARG,
                     "every shard but the last needs a width that is a multiple of %d (got Vs = %d)",
                     SV_SHARD_ALIGN, Vs);
  return SV_OK;
}

static bool aligned16(const void* q) { return reinterpret_cast<uintptr_t>(q) % 16 == 0; }

int spec_verify_shard_stats(const void* target_shard, const void* draft_shard,
                            const int32_t* draft_tokens, const float* temps, int B, int gamma,
                            int V, int v0, int Vs, int dtype, void* out_stats, void* workspace,
                            size_t workspace_bytes, void* stream) {
  const bool shape_ok = B > 0 && sizes_ok(B, gamma, Vs, dtype);
  const Layout lay = shape_ok ? layout_single(B, gamma, Vs, dtype) : Layout{};
  int rc = check_common(target_shard, draft_shard, draft_tokens, temps, B, gamma, Vs, dtype, 0,
                        out_stats, out_stats, workspace, workspace_bytes, lay.total);
  if (rc != SV_OK || B == 0) return rc;
  if ((rc = check_shard(V, v0, Vs)) != SV_OK) return rc;
  if (!aligned16(out_stats)) return set_error(SV_ERR_INVALID_ARG, "out_stats must be 16-byte aligned");
  if ((rc = check_device()) != SV_OK) return rc;
  return launch_shard_stats(target_shard, draft_shard, draft_tokens, temps, B, gamma, V, v0, Vs,
                            dtype, out_stats, workspace, lay, static_cast<cudaStream_t>(stream));
}

int spec_verify_shard_decide(const void* target_shard, const void* draft_shard,
                             const int32_t* draft_tokens, const float* temps, int B, int gamma,
                             int V, int v0, int Vs, int dtype, const void* all_stats, int nshards,
                             uint64_t seed, uint64_t step, int32_t* out_accept_len,
                             int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                             void* out_candidate, void* workspace, size_t workspace_bytes,
                             void* stream) {
  const bool shape_ok = B > 0 && sizes_ok(B, gamma, Vs, dtype);
  const Layout lay = shape_ok ? layout_single(B, gamma, Vs, dtype) : Layout{};
  int rc = check_common(target_shard, draft_shard, draft_tokens, temps, B, gamma, Vs, dtype, step,
                        out_accept_len, out_tokens, workspace, workspace_bytes, lay.total);
  if (rc != SV_OK || B == 0) return rc;
  if ((rc = check_shard(V, v0, Vs)) != SV_OK) return rc;
  if (nshards < 1 || nshards > SV_MAX_SHARDS)
    return set_error(SV_ERR_INVALID_ARG, "nshards must be in [1, %d] (got %d)", SV_MAX_SHARDS, nshards);
  if (!all_stats || !out_candidate) return set_error(SV_ERR_INVALID_ARG, "NULL shard buffer");
  if (!aligned16(all_stats) || !aligned16(out_candidate))
    return set_error(SV_ERR_INVALID_ARG, "shard buffers must be 16-byte aligned");
  if ((rc = check_device()) != SV_OK) return rc;
  return launch_shard_decide(target_shard, draft_shard, draft_tokens, temps, B, gamma, V, v0, Vs,
                             dtype, all_stats, nshards, seed, step, out_accept_len, out_tokens,
                             out_target_logp, out_draft_logp, out_candidate, workspace, lay,
                             static_cast<cudaStream_t>(stream));
}

int spec_verify_shard_pick(const void* all_candidates, int nshards, int B, int gamma,
                           int32_t* out_accept_len, int32_t* out_tokens, void* stream) {
  if (B < 0 || B > SV_MAX_BATCH)
    return set_error(SV_ERR_INVALID_ARG, "B must be in [0, %d] (got %d)", SV_MAX_BATCH, B);
  if (gamma < 1 || gamma > SV_MAX_GAMMA)
    return set_error(SV_ERR_INVALID_ARG, "draft length must be in [1, %d] (got %d)", SV_MAX_GAMMA, gamma);
  if (nshards < 1 || nshards > SV_MAX_SHARDS)
    return set_error(SV_ERR_INVALID_ARG, "nshards must be in [1, %d] (got %d)", SV_MAX_SHARDS, nshards);
  if (B == 0) return SV_OK;
  if (!all_candidates || !out_accept_len || !out_tokens)
    return set_error(SV_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(all_candidates))
    return set_error(SV_ERR_INVALID_ARG, "all_candidates must be 16-byte aligned");
  int rc;
  if ((rc = check_device()) != SV_OK) return rc;
  return launch_shard_pick(all_candidates, nshards, B, gamma, out_accept_len, out_tokens,
                           static_cast<cudaStream_t>(stream));
}

static int multidraft_call(const void* target_logits, const void* draft_logits,
                           const int32_t* draft_tokens, const float* temps, int B, int K, int L,
                           int V, int dtype, int per_draft, uint64_t seed, uint64_t step,
                           int32_t* out_accept_len, int32_t* out_tokens, int32_t* out_draft_index,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (K < 1 || K > SV_MAX_DRAFTS)
    return set_error(SV_ERR_INVALID_ARG, "K must be in [1, %d] (got %d)", SV_MAX_DRAFTS, K);
  const bool shape_ok = B > 0 && sizes_ok(B, L, V, dtype);
  const Layout lay = shape_ok ? layout_multi(B, K, L, V, dtype) : Layout{};
  int rc = check_common(target_logits, draft_logits, draft_tokens, temps, B, L, V, dtype, step,
                        out_accept_len, out_tokens, workspace, workspace_bytes, lay.total);
  if (rc != SV_OK || B == 0) return rc;
  if (per_draft && K > multidraft_max_row_sets(L))
    return set_error(SV_ERR_UNSUPPORTED,
                     "per-draft rows: at most %d drafts of length %d (got K = %d)",
                     multidraft_max_row_sets(L), L, K);
  if ((rc = check_device()) != SV_OK) return rc;
  return launch_multi(target_logits, draft_logits, draft_tokens, temps, B, K, L, V, dtype,
                      per_draft, seed, step, out_accept_len, out_tokens, out_draft_index,
                      workspace, lay, static_cast<cudaStream_t>(stream));
}

int spec_verify_multidraft(const void* target_logits, const void* draft_logits,
                           const int32_t* draft_tokens, const float* temps, int B, int K, int L,
                           int V, int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                           int32_t* out_tokens, int32_t* out_draft_index, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return multidraft_call(target_logits, draft_logits, draft_tokens, temps, B, K, L, V, dtype, 0,
                         seed, step, out_accept_len, out_tokens, out_draft_index, workspace,
                         workspace_bytes, stream);
}

int spec_verify_multidraft_rows(const void* target_logits, const void* draft_logits,
                                const int32_t* draft_tokens, const float* temps, int B, int K,
                                int L, int V, int dtype, uint64_t seed, uint64_t step,
                                int32_t* out_accept_len, int32_t* out_tokens,
                                int32_t* out_draft_index, void* workspace, size_t workspace_bytes,
                                void* stream) {
  return multidraft_call(target_logits, draft_logits, draft_tokens, temps, B, K, L, V, dtype, 1,
                         seed, step, out_accept_len, out_tokens, out_draft_index, workspace,
                         workspace_bytes, stream);
}

// ------------------------------------------------------------- host buffers
namespace {
struct HostLayout {
  size_t tgt, drf, tok, tmp, acc, otok, lp, lq, ws, total;
};

HostLayout host_layout(int B, int gamma, int V, int dtype) {
  const size_t es = dtype == SV_BF16 ? 2 : 4;
  HostLayout h{};
  size_t off = 0;
  h.ws = off;  // the workspace (with its counter header) sits at offset 0
  off += layout_single(B, gamma, V, dtype).total;
  h.tgt = off;
  off += up(static_cast<size_t>(B) * (gamma + 1) * static_cast<size_t>(V) * es);
  h.drf = off;
  off += up(static_cast<size_t>(B) * gamma * static_cast<size_t>(V) * es);
  h.tok = off;
  off += up(static_cast<size_t>(B) * gamma * 4);
  h.tmp = off;
  off += up(static_cast<size_t>(B) * 4);
  h.acc = off;
  off += up(static_cast<size_t>(B) * 4);
  h.otok = off;
  off += up(static_cast<size_t>(B) * (gamma + 1) * 4);
  h.lp = off;
  off += up(static_cast<size_t>(B) * gamma * 4);
  h.lq = off;
  off += up(static_cast<size_t>(B) * gamma * 4);
  h.total = off;
  return h;
}
}  // namespace

size_t spec_verify_host_staging_size(int B, int gamma, int V, int dtype) {
  if (!sizes_ok(B, gamma, V, dtype)) return 0;
  return host_layout(B, gamma, V, dtype).total;
}

// The host-buffer path without the final synchronisation: copies in, the
// verification, copies out, all enqueued on `stream`.
static int host_enqueue(const void* target_logits, const void* draft_logits,
                        const int32_t* draft_tokens, const float* temps, int B, int gamma, int V,
                        int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                        int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                        void* staging, size_t staging_bytes, cudaStream_t s) {
  if (B < 0 || !sizes_ok(B, gamma, V, dtype))
    return check_common(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, step,
                        out_accept_len, out_tokens, staging, staging_bytes, 0);
  if (B == 0) return SV_OK;
  const HostLayout h = host_layout(B, gamma, V, dtype);
  if (!target_logits || !draft_logits || !draft_tokens || !temps || !out_accept_len || !out_tokens)
    return set_error(SV_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!staging || reinterpret_cast<uintptr_t>(staging) % 256)
    return set_error(SV_ERR_WORKSPACE, "staging buffer NULL or not 256-byte aligned");
  if (staging_bytes < h.total)
    return set_error(SV_ERR_WORKSPACE, "staging too small: %zu < %zu bytes", staging_bytes, h.total);
  if (step >> 32) return set_error(SV_ERR_INVALID_ARG, "step must be < 2^32");
  int rc = check_device();
  if (rc != SV_OK) return rc;
  char* st = static_cast<char*>(staging);
  const size_t es = dtype == SV_BF16 ? 2 : 4;
  const size_t nt = static_cast<size_t>(B) * (gamma + 1) * static_cast<size_t>(V) * es;
  const size_t nd = static_cast<size_t>(B) * gamma * static_cast<size_t>(V) * es;
  const size_t nx = static_cast<size_t>(B) * gamma * 4;
  cudaError_t e = cudaMemcpyAsync(st + h.tgt, target_logits, nt, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st + h.drf, draft_logits, nd, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(st + h.tok, draft_tokens, nx, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st + h.tmp, temps, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "host->device copy: %s", cudaGetErrorString(e));
  rc = launch_single(st + h.tgt, st + h.drf, reinterpret_cast<const int32_t*>(st + h.tok),
                     reinterpret_cast<const float*>(st + h.tmp), B, gamma, V, dtype, seed, step,
                     reinterpret_cast<int32_t*>(st + h.acc), reinterpret_cast<int32_t*>(st + h.otok),
                     out_target_logp ? reinterpret_cast<float*>(st + h.lp) : nullptr,
                     out_draft_logp ? reinterpret_cast<float*>(st + h.lq) : nullptr, st + h.ws,
                     layout_single(B, gamma, V, dtype), s);
  if (rc != SV_OK) return rc;
  e = cudaMemcpyAsync(out_accept_len, st + h.acc, static_cast<size_t>(B) * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out_tokens, st + h.otok, static_cast<size_t>(B) * (gamma + 1) * 4,
                        cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && out_target_logp)
    e = cudaMemcpyAsync(out_target_logp, st + h.lp, nx, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && out_draft_logp)
    e = cudaMemcpyAsync(out_draft_logp, st + h.lq, nx, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "device->host copy: %s", cudaGetErrorString(e));
  return SV_OK;
}

int spec_verify_host(const void* target_logits, const void* draft_logits,
                     const int32_t* draft_tokens, const float* temps, int B, int gamma, int V,
                     int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                     int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                     void* staging, size_t staging_bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rc = host_enqueue(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype,
                              seed, step, out_accept_len, out_tokens, out_target_logp,
                              out_draft_logp, staging, staging_bytes, s);
  if (rc != SV_OK || B == 0) return rc;
  const cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return set_error(SV_ERR_CUDA, "device->host copy: %s", cudaGetErrorString(e));
  return SV_OK;
}

int spec_verify_host_async(const void* target_logits, const void* draft_logits,
                           const int32_t* draft_tokens, const float* temps, int B, int gamma,
                           int V, int dtype, uint64_t seed, uint64_t step,
                           int32_t* out_accept_len, int32_t* out_tokens, float* out_target_logp,
                           float* out_draft_logp, void* staging, size_t staging_bytes,
                           void* stream) {
  return host_enqueue(target_logits, draft_logits, draft_tokens, temps, B, gamma, V, dtype, seed,
                      step, out_accept_len, out_tokens, out_target_logp, out_draft_logp, staging,
                      staging_bytes, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
