/*
 * spec_verify_shard.h -- vocabulary-sharded single-draft verification.
 *
 * The same verification as spec_verify (FlashSpec, Methodology s.1; FlexDraft,
 * Problem definition; Speculative Speculative Decoding, s.2 Saguaro sampling),
 * for logits split over the vocabulary as a tensor-parallel LM head leaves
 * them: rank r of n holds columns [v0_r, v0_r + Vs_r) of every target and
 * draft row, [B, gamma + 1, Vs_r] and [B, gamma, Vs_r].  The pages verify on
 * one device; the split is this library's, and its results are those of
 * spec_verify on the whole rows (the same Philox streams, keyed by global
 * vocabulary and group indices), up to fp32 rounding of the row sums.
 *
 * Shards: v0_r is a multiple of SV_SHARD_ALIGN (1024, the width of a race
 * group, so no group straddles two ranks), shards do not overlap, and
 * together they cover [0, V).  Every shard but the last (v0 + Vs == V) has a
 * width that is a multiple of SV_SHARD_ALIGN.
 *
 * One verification is three calls on every rank, with two exchanges that
 * the caller makes (an all-gather, e.g. ncclAllGather, over the n ranks in
 * rank order):
 *
 *   1. spec_verify_shard_stats: per (sequence, position) the shard's
 *      statistics of the target and draft row (maximum, scaled softmax sum or
 *      first argmax with a global index) and the draft token's two logits
 *      when this shard holds that token.
 *      -> all-gather the n records into one buffer, rank r's at offset
 *         r * spec_verify_shard_stats_bytes(B, gamma).
 *   2. spec_verify_shard_decide: every rank merges the n records (in
 *      buffer order, so every rank reaches bit-identical row statistics),
 *      takes the acceptance decision, writes accept_len, the accepted
 *      tokens and the log-probabilities, and runs the two-level race of the
 *      correction / bonus draw over its own groups: level 1 over the shard's
 *      1024-entry groups, level 2 inside the shard's best group.  Writes
 *      one race candidate per sequence (the shard's best group, its weight,
 *      its exponential and its level-2 token).  A shard whose residual
 *      weights are all zero writes its candidate of the race over p_j
 *      instead (the draw from p_j when the whole residual vanishes).
 *      -> all-gather the n candidate arrays likewise.
 *   3. spec_verify_shard_pick: the winning candidate over the ranks (largest
 *      w / E, lowest group index on ties; the candidates of the race over
 *      p_j only when no rank has residual weight) gives the drawn token,
 *      written at out_tokens[b][accept_len[b]].
 *
 * Every rank ends with the same outputs.  Conventions (streams, errors,
 * device-data problems, the workspace header, bounded waits) are those of
 * spec_verify.h.  The workspace of a rank is spec_verify_workspace_size(B,
 * gamma, Vs, dtype) bytes, zeroed once; calls 1 and 2 of one verification
 * use the same workspace, on one stream.
 */
#ifndef SPEC_VERIFY_SHARD_H
#define SPEC_VERIFY_SHARD_H

#include <stddef.h>
#include <stdint.h>

#include "spec_verify.h"

#ifdef __cplusplus
extern "C" {
#endif

#define SV_SHARD_ALIGN 1024
#define SV_MAX_SHARDS 256

/* Bytes of one rank's statistics record: B (gamma + 1) x 48 (per position:
 * the target row's {max, sum, reference exponent or argmax, NaN flag} as
 * four 32-bit words, the draft row's likewise, then the draft token's target
 * and draft logit (NaN where this shard does not hold the token) and two
 * zero words).  0 for sizes out of range. */
size_t spec_verify_shard_stats_bytes(int B, int gamma);

/* Bytes of one rank's candidate array: B x 32 ({w, E} fp32, the global
 * group index, the token, the kind (0 no draw, 1 the draw law, 2 the race
 * over p_j of a shard whose residual vanished), the draw position j, two
 * zero words).  0 for sizes out of range. */
size_t spec_verify_shard_candidate_bytes(int B);

/* Call 1.  target_shard [B][gamma + 1][Vs], draft_shard [B][gamma][Vs]
 * (device, dtype, dense), draft_tokens [B][gamma] global token ids,
 * temps [B]; V the full vocabulary, v0 / Vs this shard.  out_stats: device,
 * 16-byte aligned, spec_verify_shard_stats_bytes(B, gamma) bytes (written
 * in full). */
int spec_verify_shard_stats(const void* target_shard, const void* draft_shard,
                            const int32_t* draft_tokens, const float* temps, int B, int gamma,
                            int V, int v0, int Vs, int dtype, void* out_stats, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Call 2.  The shard's logits and the sequence inputs as in call 1;
 * all_stats: the n records of call 1 gathered in rank order (device,
 * 16-byte aligned, n x spec_verify_shard_stats_bytes(B, gamma) bytes), the
 * same buffer contents on every rank.  Outputs as spec_verify's, except that
 * out_tokens[b][accept_len[b]] stays -1 until call 3 (greedy sequences: the
 * target argmax, written here); out_target_logp / out_draft_logp may be
 * NULL.  out_candidate: device, 16-byte aligned,
 * spec_verify_shard_candidate_bytes(B) bytes (written in full). */
int spec_verify_shard_decide(const void* target_shard, const void* draft_shard,
                             const int32_t* draft_tokens, const float* temps, int B, int gamma,
                             int V, int v0, int Vs, int dtype, const void* all_stats, int nshards,
                             uint64_t seed, uint64_t step, int32_t* out_accept_len,
                             int32_t* out_tokens, float* out_target_logp, float* out_draft_logp,
                             void* out_candidate, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Call 3.  all_candidates: the n candidate arrays of call 2 gathered in
 * rank order (device, 16-byte aligned); out_accept_len [B] and out_tokens
 * [B][gamma + 1] as left by call 2.  Candidates whose ranks disagree on the
 * draw (ranks given different sequence inputs, or records gathered in
 * different orders) mark the sequence as spec_verify marks invalid data:
 * accept_len -1, tokens -1, on every rank.  Needs no workspace. */
int spec_verify_shard_pick(const void* all_candidates, int nshards, int B, int gamma,
                           int32_t* out_accept_len, int32_t* out_tokens, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_SHARD_H */
