// sv_internal.h -- shared host/device declarations of the verifier library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "spec_verify.h"

namespace sv {

constexpr int kMaxRowsPerSeq = 2 * SV_MAX_GAMMA + 1;

// Per-sequence hand-off from the decision to the draw.
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

// Draw partial: best exponential-race candidate of one chunk.
struct alignas(16) RacePartial {
  float w;
  float e;
  int idx;
  int pad;
};

// Vocabulary shards: one rank's race candidate for sequence b (32 bytes,
// the layout spec_verify_shard.h documents).
enum ShardKind { kShardNoDraw = 0, kShardDrawLaw = 1, kShardTargetRace = 2 };
struct alignas(16) ShardCand {
  float w;      // the shard's best group weight (0: no mass in this shard)
  float e;      // its exponential
  int group;    // its global group index
  int token;    // the level-2 winner inside that group (-1: none)
  int kind;     // ShardKind
  int j;        // draw position
  int pad0, pad1;
};
static_assert(sizeof(ShardCand) == 32, "candidate record is 32 bytes");

// Inputs, outputs and decision state of a single-draft call.
struct CallParams {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const float* temps;
  int B, gamma, V, rps;  // rps = 2 gamma + 1 rows per sequence
  uint64_t seed;
  uint32_t step;
  unsigned* ticket;     // [B] row arrivals
  SeqInfo* info;        // [B] decision -> draw hand-off
  int32_t* accept_len;
  int32_t* out_tokens;
  float* out_lp;
  float* out_lq;
};

// Workspace layout of one call.  A header of fixed size at offset 0 holds the
// per-sequence arrival counters (one slot per sequence, up to SV_MAX_BATCH),
// so their positions do not depend on the shape: every call leaves them at
// zero and a later call of any shape finds them zeroed.  Header: three u32
// arrays, the row kernel's arrivals, the draw kernel's arrivals and the
// decision-published flags.
constexpr size_t kSeqSlots = static_cast<size_t>(SV_MAX_BATCH) * sizeof(unsigned);
constexpr size_t kHeaderBytes = 3 * kSeqSlots;

struct Layout {
  size_t part1, ticket1, info, part2, ticket2, ready, resid, total;
  int nc, nc2;
};

Layout layout_single(int B, int gamma, int V, int dtype);
int draw_chunks(int V);  // bound on draw CTAs per sequence (sv_single.cu)
int row_segments(int V, int dtype);  // bound on row segments per row (sv_single.cu)
Layout layout_multi(int B, int K, int L, int V, int dtype);
// Small batches (sv_small.cu): whether a shape takes the one-cluster-per-
// sequence kernel, and its launch.
bool small_path(int B, int gamma, int V, int dtype);
int launch_small(const CallParams& p1, int dtype, cudaStream_t stream);
size_t multidraft_global_bytes(int B, int V);  // residual laws of the multi-draft kernel (sv_multi.cu)

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
                 const float* temps, int B, int K, int L, int V, int dtype, int per_draft,
                 uint64_t seed, uint64_t step, int32_t* out_accept_len, int32_t* out_tokens,
                 int32_t* out_draft_index, void* workspace, const Layout& lay,
                 cudaStream_t stream);
int multidraft_max_row_sets(int L);  // largest K with a row set per draft (sv_multi.cu)

// Vocabulary-sharded single draft (sv_single.cu).  The target / draft
// pointers are the shard's [B][gamma + 1][Vs] / [B][gamma][Vs] rows.
int launch_shard_stats(const void* target, const void* draft, const int32_t* tokens,
                       const float* temps, int B, int gamma, int V, int v0, int Vs, int dtype,
                       void* out_stats, void* workspace, const Layout& lay, cudaStream_t stream);
int launch_shard_decide(const void* target, const void* draft, const int32_t* tokens,
                        const float* temps, int B, int gamma, int V, int v0, int Vs, int dtype,
                        const void* all_stats, int nshards, uint64_t seed, uint64_t step,
                        int32_t* out_accept_len, int32_t* out_tokens, float* out_lp,
                        float* out_lq, void* out_candidate, void* workspace, const Layout& lay,
                        cudaStream_t stream);
int launch_shard_pick(const void* all_candidates, int nshards, int B, int gamma,
                      int32_t* out_accept_len, int32_t* out_tokens, cudaStream_t stream);

}  // namespace sv
