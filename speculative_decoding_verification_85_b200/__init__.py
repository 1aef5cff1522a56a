"""B200 (sm_100a) batched speculative-sampling verification.

The hot path is the C-ABI library ``libspecverify.so`` (hand-written CUDA
kernels, ``include/spec_verify.h``); this package is a thin ctypes binding
that marshals torch tensors (device memory, the current stream) into that ABI.
It performs no computation of its own and has no CPU fallback: importing it
without the built library, or calling it on tensors that are not on a CUDA
device, raises.  The same library holds the host-side draft selector
(``include/sv_bandit.h``, native C++), bound here as ``Bandit``.
"""
from ._binding import (  # noqa: F401
    BF16, F32, SHARD_ALIGN, Bandit, SpecVerifyError, Verifier, gather_records, lib, library_path,
    multidraft_workspace_size, shard_candidate_bytes, shard_stats_bytes, spec_verify,
    spec_verify_host, spec_verify_multidraft, spec_verify_noalloc,
    spec_verify_noalloc_max_workspace, spec_verify_shard_decide, spec_verify_shard_pick,
    spec_verify_shard_stats, spec_verify_vocab_sharded, staging_size, vocab_shards,
    workspace_size,
)

__all__ = [
    "spec_verify", "spec_verify_multidraft", "spec_verify_host", "Verifier", "workspace_size",
    "multidraft_workspace_size", "staging_size", "SpecVerifyError", "lib", "library_path",
    "spec_verify_noalloc", "spec_verify_noalloc_max_workspace", "Bandit",
    "spec_verify_shard_stats", "spec_verify_shard_decide", "spec_verify_shard_pick",
    "spec_verify_vocab_sharded", "vocab_shards", "shard_stats_bytes", "shard_candidate_bytes",
    "gather_records", "SHARD_ALIGN",
]
