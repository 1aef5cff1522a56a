// sv_internal.h -- shared host/device declarations of the verifier library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "spec_verify.h"

namespace sv {

constexpr int kP1Threads = 256;   // pass-1 CTA size
constexpr int kP2Threads = 256;   // pass-2 CTA size
constexpr int kMdThreads = 1024;  // multi-draft sequential kernel CTA size
constexpr int kMaxRowsPerSeq = 2 * SV_MAX_GAMMA + 1;

// Partial of one (row, chunk): raw max, scaled sum, index slot, NaN seen; 16
// bytes, stored as one vector.  The multi-draft chunk pass keeps
// s = sum 2^{(z - max) c} and the first argmax index (greedy rows); the
// single-draft row kernel keeps S = sum 2^{z c - R} against an integer
// reference R, carried as float bits in the index slot (softmax rows), or
// the first argmax index (greedy rows).
struct alignas(16) RowPartial {
  float m;
  float s;
  int arg;
  int bad;
};

// Per-sequence hand-off from the decision to pass 2.
struct alignas(16) SeqInfo {
  int mode;     // kModeNone / kModeResidual / kModeBonus
  int j;        // position of the draw
  float zmp;    // raw max of target row j
  float zmq;    // raw max of draft row j (residual)
  float c;      // log2(e) / T
  float lsp;    // log2 of the target row's scaled sum: p_v = 2^{(z_v - zmp) c - lsp}
  float lsq;    // log2 of the draft row's scaled sum
  float pad;
};

// Pass-2 partial: best exponential-race candidate of one chunk.
struct alignas(16) RacePartial {
  float w;
  float e;
  int idx;
  int pad;
};

struct Pass1Params {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const float* temps;
  int B, gamma, V, nc, rps;  // gamma = L for multi-draft; rps = 2 gamma + 1
  uint64_t seed;
  uint32_t step;
  RowPartial* part;     // [B * rps * nc]
  unsigned* ticket;     // [B]
  RowPartial* rowstat;  // [B * rps] combined rows (multi-draft)
  SeqInfo* info;        // [B] (single-draft)
  int32_t* accept_len;
  int32_t* out_tokens;
  float* out_lp;
  float* out_lq;
};

struct MdParams {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const float* temps;
  int B, K, L, V;
  uint64_t seed;
  uint32_t step;
  const RowPartial* rowstat;  // [B * (2L + 1)]
  float* R;                   // [B * V] residual law workspace
  int32_t* accept_len;
  int32_t* out_tokens;
  int32_t* out_draft_index;
};

// Workspace layout of one call.  The arrival counters live in a header of
// fixed size at offset 0 (one slot per sequence, up to SV_MAX_BATCH), so their
// position does not depend on the shape: every call leaves them at zero and a
// later call of any shape finds zeroed counters.
// Header: 256 reserved bytes (zero, unused by the current kernels), then the
// per-sequence row-kernel and draw-kernel arrival counters.
constexpr size_t kHeaderCtl = 256;
constexpr size_t kHeaderBytes = kHeaderCtl + 2 * static_cast<size_t>(SV_MAX_BATCH) * sizeof(unsigned);

struct Layout {
  size_t ctl, part1, ticket1, info, rowstat, part2, ticket2, resid, total;
  int nc, nc2;
};

Layout layout_single(int B, int gamma, int V, int dtype);
int draw_chunks(int V, int dtype);   // bound on draw CTAs per sequence (sv_single.cu)
int row_segments(int V, int dtype);  // bound on row segments per row (sv_single.cu)
Layout layout_multi(int B, int K, int L, int V, int dtype);

// Host helpers (sv_api.cu).
int set_error(int status, const char* fmt, ...);
int check_device();
int check_launch(const char* what);

// Kernel launchers (sv_single.cu / sv_multi.cu).
int launch_single(const void* target, const void* draft, const int32_t* tokens,
                  const float* temps, int B, int gamma, int V, int dtype, uint64_t seed,
                  uint64_t step, int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                  float* out_lq, void* workspace, const Layout& lay, cudaStream_t stream);
int launch_multi(const void* target, const void* draft, const int32_t* tokens,
                 const float* temps, int B, int K, int L, int V, int dtype, uint64_t seed,
                 uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                 int32_t* out_draft_index, void* workspace, const Layout& lay,
                 cudaStream_t stream);

}  // namespace sv
