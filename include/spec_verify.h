/*
 * spec_verify.h -- C ABI of the B200 (sm_100a) speculative-sampling verifier.
 *
 * Operations (page title, section):
 *   spec_verify            "FlashSpec: Adaptive Speculative Decoding with Online
 *                          Bandit Draft Selection and Triton-Optimised
 *                          Verification", Methodology s.1 (on-device
 *                          accept/reject, temperature before the log-softmax,
 *                          log-space arithmetic); "FlexDraft", Problem definition
 *                          (correction token drawn at the first rejection);
 *                          "Speculative Speculative Decoding", s.2 Saguaro
 *                          sampling (residual r proportional to
 *                          max(p_target - p_draft, 0)).
 *   spec_verify_multidraft "SpecTr-GBV: Multi-Draft Block Verification
 *                          Accelerating Speculative Decoding", Methodology,
 *                          Algorithm 1.
 *   spec_verify_shard_*    spec_verify for logits split over the vocabulary
 *                          across ranks (spec_verify_shard.h).
 *
 * Conventions shared by every entry point
 *   - Logit tensors are dense, row-major, contiguous, in device memory, fp32
 *     or bf16 (sv_dtype).  Any V >= 1 and any base alignment of the element
 *     type are accepted.
 *   - temps[b] is the sampling temperature of sequence b (device fp32).
 *     temps[b] == 0 selects greedy verification (argmax matching).
 *   - Randomness: Philox4x32-10 (Salmon et al., SC'11) with key
 *     (lo32(seed), hi32(seed)) and counter (c0, b, lo32(step), tag<<24 | k<<12
 *     | pos).  Acceptance uniform of position i: tag 1, c0 = i, word 0,
 *     u = (x >> 8) * 2^-24.  The single-draft correction/bonus token at
 *     position j is drawn by a two-level exponential race over the weights
 *     w_v (max(p_j - q_j, 0), or p_gamma): vocabulary groups of 1024 entries
 *     race with their summed weights, group g with the exponential
 *     E = -ln U of tag 7, c0 = g, word 0; within the winning group entry v
 *     races with tag 2, c0 = v >> 2, word v & 3; U = (2 (x >> 9) + 1) 2^-24
 *     in both; the largest w / E wins (lowest index on ties).  Multi-draft
 *     uses tag 3 (k = draft index, pos = i) for its acceptance uniforms and
 *     the per-entry race with tag 4 for its correction token.  Every step
 *     therefore replays bit-exactly from (inputs, seed, step).
 *   - Asynchronous: every entry point enqueues work on `stream` (a
 *     cudaStream_t; NULL is the legacy default stream) and returns without
 *     synchronising.  Results are valid once the stream has reached that
 *     point.  Nothing is allocated during a call and no state is kept
 *     between calls except inside the caller's workspace.
 *   - Workspace: caller-owned device memory of at least the size returned by
 *     the matching *_workspace_size function, 256-byte aligned, zero-filled
 *     before its first use (spec_verify_workspace_init or cudaMemset).  The
 *     workspace starts with a fixed 768 KB header of per-sequence arrival
 *     counters and flags (their offsets do not depend on the shape), followed by
 *     per-call partial results.  Every call returns the counters to zero, so
 *     the workspace can be reused by later calls on the same stream, of any
 *     shape that fits, without clearing.  Two calls that may run concurrently
 *     (different streams) need different workspaces.
 *   - Errors: a host-checkable problem (NULL pointer, a size out of range, an
 *     unknown dtype, step >= 2^32, a workspace that is too small or
 *     misaligned, a device other than sm_100) returns a non-zero sv_status and
 *     launches nothing; spec_verify_last_error() then describes it.  Problems
 *     that live in device data (temps[b] negative, NaN or infinite; a draft
 *     token outside [0, V); a logit row whose maximum is NaN, +inf, or -inf)
 *     mark only that sequence: accept_len[b] = -1 and all its tokens -1.  The
 *     kernels never trap; every wait on another CTA is bounded in time (two
 *     seconds), and a wait that runs out marks its sequence the same way.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SV_F32 = 0, SV_BF16 = 1 } sv_dtype;

typedef enum {
  SV_OK = 0,
  SV_ERR_INVALID_ARG = 1, /* bad pointer, size, dtype or step              */
  SV_ERR_UNSUPPORTED = 2, /* not an sm_100 device                          */
  SV_ERR_CUDA = 3,        /* a CUDA runtime call or a launch failed        */
  SV_ERR_WORKSPACE = 4    /* workspace NULL, too small or misaligned       */
} sv_status;

/* Largest draft length (gamma or L), draft count (K) and batch (B) accepted. */
#define SV_MAX_GAMMA 64
#define SV_MAX_DRAFTS 32
#define SV_MAX_BATCH 65536

/* Library version, (major << 16) | minor. */
int spec_verify_version(void);

/* Message for the last non-OK status returned on the calling host thread. */
const char* spec_verify_last_error(void);

/* Bytes of workspace spec_verify needs for this shape (0 on bad sizes). */
size_t spec_verify_workspace_size(int B, int gamma, int V, int dtype);

/* Zero-fill a workspace on `stream` (cudaMemsetAsync). */
int spec_verify_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * spec_verify -- single-draft verification of a batch of B sequences.
 *
 * Inputs (device):
 *   target_logits [B, gamma+1, V]  target-model logits at the gamma draft
 *                                  positions and the one after them.
 *   draft_logits  [B, gamma, V]    draft-model logits at the gamma positions.
 *   draft_tokens  [B, gamma] int32 the proposed tokens.
 *   temps         [B] fp32         per-sequence temperature (0 = greedy).
 * Outputs (device, written by the call):
 *   out_accept_len [B] int32        j = number of accepted draft tokens, or -1.
 *   out_tokens     [B, gamma+1]     x_0..x_{j-1}, then the correction token
 *                                   (residual draw at j < gamma, bonus draw
 *                                   from the target row gamma at j == gamma),
 *                                   then -1 padding.
 *   out_target_logp, out_draft_logp [B, gamma] fp32 or NULL: the gathered
 *                                   log-probabilities log_softmax(z/T)[x_i]
 *                                   (NaN at T = 0 and for invalid sequences).
 * Per sequence (T > 0): s_v = fl32(z_v / T) per row; a draft token is
 * accepted when u_i < min(1, exp(lp_i - lq_i)); j is the first rejection;
 * the correction token is argmax_v (log max(p_j - q_j, 0)_v + G_v), or
 * argmax_v (lp_gamma,v + G_v) when every token was accepted.  At T = 0 a
 * token is accepted when it equals the first argmax of the raw target row,
 * and the correction token is that argmax at j.
 */
int spec_verify(const void* target_logits, const void* draft_logits,
                const int32_t* draft_tokens, const float* temps, int B, int gamma, int V,
                int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace spec_verify_multidraft needs (0 on bad sizes). */
size_t spec_verify_multidraft_workspace_size(int B, int K, int L, int V, int dtype);

/*
 * spec_verify_multidraft -- K i.i.d. draft blocks of length L per sequence,
 * greedy sub-block acceptance with a rejected set H (SpecTr-GBV, Algorithm 1).
 *
 * Inputs (device): target_logits [B, L+1, V]; draft_logits [B, L, V] shared
 * by the K drafts (position-wise draft law); draft_tokens [B, K, L] int32;
 * temps [B].
 * Outputs (device): out_accept_len [B] (tau, or -1); out_tokens [B, L+1]
 * (the accepted prefix of draft a, the correction token at tau, -1 padding);
 * out_draft_index [B] (a, -1 when tau == 0; may be NULL).
 * The acceptance weights are the greedy block-verification ones
 * (w, h = A / (A + 1 - w), A = sum_v max(w P_{i+1} - Q_{i+1}, 0)); drafts are
 * visited in index order; a draft whose token at tau was rejected before is
 * skipped, and the draft law at tau is conditioned on not being in H.  At
 * T = 0 the accepted block is the longest draft prefix that matches the
 * target argmaxes.
 */
int spec_verify_multidraft(const void* target_logits, const void* draft_logits,
                           const int32_t* draft_tokens, const float* temps, int B, int K,
                           int L, int V, int dtype, uint64_t seed, uint64_t step,
                           int32_t* out_accept_len, int32_t* out_tokens,
                           int32_t* out_draft_index, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * spec_verify_multidraft_rows -- multi-draft verification with a row set per
 * draft, the prefix-conditioned use of SpecTr-GBV (Methodology, Algorithm 1:
 * K i.i.d. draft sequences, each verified against the target's
 * distributions after its own prefix).
 *
 * Inputs (device): target_logits [B, K, L+1, V] -- row (k, i) holds the
 * target logits after draft k's own prefix x_k[0..i); draft_logits
 * [B, K, L, V] likewise; draft_tokens [B, K, L]; temps [B].  Outputs and
 * workspace (spec_verify_multidraft_workspace_size) as spec_verify_multidraft.
 * Draft k is weighed with its own rows; the residual law starts from row set
 * 0 (every draft shares the empty prefix) and, after an advance, comes from
 * the accepted draft's rows; the whole-block correction is drawn from row L
 * of the accepted draft.  With K equal copies of one row set the results are
 * those of spec_verify_multidraft.  K (2L + 1) must not exceed 256 (row
 * statistics kept per sequence): larger shapes return SV_ERR_UNSUPPORTED.
 */
int spec_verify_multidraft_rows(const void* target_logits, const void* draft_logits,
                                const int32_t* draft_tokens, const float* temps, int B, int K,
                                int L, int V, int dtype, uint64_t seed, uint64_t step,
                                int32_t* out_accept_len, int32_t* out_tokens,
                                int32_t* out_draft_index, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * spec_verify_host -- spec_verify on HOST buffers, for callers whose logits
 * live in host memory.  The inputs are copied host->device into `staging`
 * (device memory, at least spec_verify_host_staging_size bytes, 256-byte
 * aligned; it begins with the workspace, so it must be zero-filled before
 * its first use), verified, and the outputs copied back device->host; the
 * call returns after `stream` has finished those copies.  Host buffers
 * should be pinned for asynchronous copies.  out_*_logp may be NULL.
 */
size_t spec_verify_host_staging_size(int B, int gamma, int V, int dtype);
int spec_verify_host(const void* target_logits, const void* draft_logits,
                     const int32_t* draft_tokens, const float* temps, int B, int gamma,
                     int V, int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                     int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                     void* staging, size_t staging_bytes, void* stream);

/*
 * spec_verify_host_async -- spec_verify_host without the final
 * synchronisation: the input copies, the verification and the output copies
 * are enqueued on `stream` and the call returns; the host outputs are valid
 * once the stream has reached that point.  With pinned host buffers, two
 * staging buffers used on two streams in turn let one step's upload overlap
 * the previous step's verification and download.  A staging buffer must not
 * be reused before the work enqueued on it has finished (order it on its
 * stream); the argument checks and errors are those of spec_verify_host.
 */
int spec_verify_host_async(const void* target_logits, const void* draft_logits,
                           const int32_t* draft_tokens, const float* temps, int B, int gamma,
                           int V, int dtype, uint64_t seed, uint64_t step,
                           int32_t* out_accept_len, int32_t* out_tokens, float* out_target_logp,
                           float* out_draft_logp, void* staging, size_t staging_bytes,
                           void* stream);

/*
 * spec_verify_noalloc -- spec_verify for callers that cannot allocate device
 * memory at verification time (an engine that reserves almost all of the
 * GPU's memory up front for weights and KV cache, or a decode path that must
 * never enter an allocator).  Not an operation of the source pages: it is
 * spec_verify with the same inputs, outputs and results, but the scratch
 * space comes from a fixed array of SV_NOALLOC_MAX_WORKSPACE bytes in the
 * library's own device memory (one per device, present once the library is
 * loaded) instead of a caller workspace.  The call allocates nothing.
 *   - Size limit: shapes whose spec_verify_workspace_size exceeds
 *     SV_NOALLOC_MAX_WORKSPACE (8 MiB; for example B = 256, gamma = 4,
 *     V = 151936 bf16 needs about 1.5 MB) return SV_ERR_WORKSPACE and launch
 *     nothing; use spec_verify with a caller workspace for those.
 *   - First call per device: it looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and clears its counter
 *     header on `stream`.  Make that first call before any stream capture.
 *   - Concurrency: all calls on one device share the array, so two calls
 *     that may overlap on the GPU (different streams without ordering) race
 *     and their results are undefined.  Order them on one stream.
 */
#define SV_NOALLOC_MAX_WORKSPACE (8u << 20)
size_t spec_verify_noalloc_max_workspace(void);
int spec_verify_noalloc(const void* target_logits, const void* draft_logits,
                        const int32_t* draft_tokens, const float* temps, int B, int gamma,
                        int V, int dtype, uint64_t seed, uint64_t step, int32_t* out_accept_len,
                        int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                        void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SPEC_VERIFY_H */
