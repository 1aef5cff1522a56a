"""CPU checks of the C-ABI library: it loads without a GPU and exports every
function that include/spec_verify.h declares; size queries work; calls fail
loudly (no CPU fallback) when there is no device."""
import ctypes
import os
import re

import pytest

import speculative_decoding_verification_85_b200 as sv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert "spec_verify" in names and "spec_verify_multidraft" in names
    lib = ctypes.CDLL(sv.library_path)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_size_queries():
    assert sv.lib().spec_verify_version() >> 16 == 1
    assert sv.workspace_size(256, 4, 151936, sv.BF16) > 0
    assert sv.workspace_size(1, 0, 10, sv.BF16) == 0      # gamma out of range
    assert sv.workspace_size(1, 65, 10, sv.BF16) == 0
    assert sv.workspace_size(1, 4, 10, 7) == 0            # unknown dtype
    assert sv.multidraft_workspace_size(8, 4, 5, 32000, sv.BF16) > 0
    assert sv.multidraft_workspace_size(8, 33, 5, 32000, sv.BF16) == 0
    assert sv.staging_size(16, 5, 32000, sv.BF16) > 16 * 11 * 32000 * 2


def test_host_side_argument_errors():
    L = sv.lib()
    # B = 0 is a no-op; bad sizes are rejected before any CUDA call
    assert L.spec_verify(None, None, None, None, 0, 4, 10, 1, 0, 0, None, None, None, None,
                         None, 0, None) == 0
    assert L.spec_verify(None, None, None, None, 1, 0, 10, 1, 0, 0, None, None, None, None,
                         None, 0, None) == 1
    assert b"draft length" in L.spec_verify_last_error()
    assert L.spec_verify(None, None, None, None, 1, 4, 10, 1, 0, 2**32, None, None, None,
                         None, None, 0, None) == 1
    assert L.spec_verify_multidraft(None, None, None, None, 1, 0, 4, 10, 1, 0, 0, None, None,
                                    None, None, 0, None) == 1


def test_cpu_tensors_rejected():
    import torch
    t = torch.zeros(1, 3, 8)
    with pytest.raises(ValueError, match="CUDA"):
        sv.spec_verify(t, torch.zeros(1, 2, 8), torch.zeros(1, 2, dtype=torch.int32),
                       torch.ones(1))


def test_noalloc_rejects_shapes_beyond_its_fixed_workspace():
    """Host-side check, before any CUDA call: a shape whose workspace exceeds
    the fixed array is refused with SV_ERR_WORKSPACE."""
    L = sv.lib()
    assert sv.spec_verify_noalloc_max_workspace() == 8 << 20
    B, g, V = 2048, 8, 128256
    assert sv.workspace_size(B, g, V, sv.BF16) > sv.spec_verify_noalloc_max_workspace()
    rc = L.spec_verify_noalloc(None, None, None, None, B, g, V, sv.BF16, 0, 0, None, None, None,
                               None, None)
    assert rc == 4
    assert b"fixed" in L.spec_verify_last_error()


def test_noalloc_reports_bad_shapes_before_any_device_setup():
    """A bad shape (gamma out of range) is reported as SV_ERR_INVALID_ARG, as
    spec_verify reports it: the no-alloc entry point neither looks up its
    fixed array nor queues its first-call clear (no CUDA device is needed)."""
    L = sv.lib()
    for g in (0, 65):
        rc = L.spec_verify_noalloc(None, None, None, None, 1, g, 100, sv.BF16, 0, 0, None, None,
                                   None, None, None)
        assert rc == 1
        assert b"draft length" in L.spec_verify_last_error()
    rc = L.spec_verify_noalloc(None, None, None, None, 1, 4, 100, 9, 0, 0, None, None, None,
                               None, None)
    assert rc == 1 and b"dtype" in L.spec_verify_last_error()


def test_shard_sizes_and_host_side_checks():
    """Vocabulary shards: record sizes, and the shard rules checked on the
    host before any CUDA call (the pointers below are never dereferenced)."""
    L = sv.lib()
    assert sv.shard_stats_bytes(4, 3) == 4 * 4 * 48
    assert sv.shard_candidate_bytes(5) == 5 * 32
    assert sv.shard_stats_bytes(1, 0) == 0 and sv.shard_candidate_bytes(-1) == 0
    fake = ctypes.c_void_p(1 << 20)
    ws_bytes = 1 << 30

    def stats(V, v0, Vs):
        return L.spec_verify_shard_stats(fake, fake, fake, fake, 2, 3, V, v0, Vs, sv.BF16, fake,
                                         fake, ws_bytes, None)

    assert stats(5000, 100, 2048) == 1
    assert b"multiple of 1024" in L.spec_verify_last_error()
    assert stats(5000, 0, 1000) == 1
    assert b"every shard but the last" in L.spec_verify_last_error()
    assert stats(5000, 4096, 1000) == 1
    assert b"must lie in" in L.spec_verify_last_error()
    assert L.spec_verify_shard_pick(fake, 0, 2, 3, fake, fake, None) == 1
    assert b"nshards" in L.spec_verify_last_error()
    assert L.spec_verify_shard_pick(None, 1, 0, 3, None, None, None) == 0  # B = 0: nothing to do


def test_vocab_shards_cover_the_vocabulary():
    for V, n in ((32000, 2), (32000, 3), (151936, 8), (128256, 4), (5000, 3), (1024, 1),
                 (1025, 2)):
        b = sv.vocab_shards(V, n)
        assert len(b) == n and b[0][0] == 0
        for (v0, Vs), (v1, _) in zip(b, b[1:]):
            assert v0 % sv.SHARD_ALIGN == 0 and Vs % sv.SHARD_ALIGN == 0 and v0 + Vs == v1
        assert b[-1][0] + b[-1][1] == V and b[-1][0] % sv.SHARD_ALIGN == 0
