"""ctypes binding of include/spec_verify.h (argument marshalling only)."""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

F32, BF16 = 0, 1
_STATUS = {0: "SV_OK", 1: "SV_ERR_INVALID_ARG", 2: "SV_ERR_UNSUPPORTED", 3: "SV_ERR_CUDA",
           4: "SV_ERR_WORKSPACE"}
_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libspecverify.so")

_lock = threading.Lock()
_lib = None


class SpecVerifyError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def lib() -> C.CDLL:
    """Load the CUDA library; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise ImportError(
                    f"{library_path} is missing: build it with "
                    "`python -m speculative_decoding_verification_85_b200.build`")
            L = C.CDLL(library_path)
            vp, i32, u64, sz = C.c_void_p, C.c_int, C.c_uint64, C.c_size_t
            L.spec_verify_version.restype = i32
            L.spec_verify_last_error.restype = C.c_char_p
            L.spec_verify_workspace_size.argtypes = [i32, i32, i32, i32]
            L.spec_verify_workspace_size.restype = sz
            L.spec_verify_multidraft_workspace_size.argtypes = [i32, i32, i32, i32, i32]
            L.spec_verify_multidraft_workspace_size.restype = sz
            L.spec_verify_workspace_init.argtypes = [vp, sz, vp]
            L.spec_verify_workspace_init.restype = i32
            L.spec_verify.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, u64, u64, vp, vp, vp, vp,
                                      vp, sz, vp]
            L.spec_verify.restype = i32
            L.spec_verify_multidraft.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, u64, u64,
                                                 vp, vp, vp, vp, sz, vp]
            L.spec_verify_multidraft.restype = i32
            L.spec_verify_multidraft_rows.argtypes = list(L.spec_verify_multidraft.argtypes)
            L.spec_verify_multidraft_rows.restype = i32
            L.spec_verify_host_staging_size.argtypes = [i32, i32, i32, i32]
            L.spec_verify_host_staging_size.restype = sz
            L.spec_verify_host.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, u64, u64, vp, vp,
                                           vp, vp, vp, sz, vp]
            L.spec_verify_host.restype = i32
            L.spec_verify_host_async.argtypes = list(L.spec_verify_host.argtypes)
            L.spec_verify_host_async.restype = i32
            L.spec_verify_noalloc_max_workspace.argtypes = []
            L.spec_verify_noalloc_max_workspace.restype = sz
            L.spec_verify_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, u64, u64, vp, vp,
                                              vp, vp, vp]
            L.spec_verify_noalloc.restype = i32
            L.sv_bandit_create.argtypes = [i32, i32, u64]
            L.sv_bandit_create.restype = vp
            L.sv_bandit_destroy.argtypes = [vp]
            L.sv_bandit_destroy.restype = None
            L.sv_bandit_select.argtypes = [vp, C.POINTER(C.c_int)]
            L.sv_bandit_select.restype = i32
            L.sv_bandit_update.argtypes = [vp, i32, C.c_double]
            L.sv_bandit_update.restype = i32
            L.sv_bandit_update_accept.argtypes = [vp, i32, vp, i32, i32]
            L.sv_bandit_update_accept.restype = i32
            L.sv_bandit_stats.argtypes = [vp, vp, vp]
            L.sv_bandit_stats.restype = i32
            L.spec_verify_shard_stats_bytes.argtypes = [i32, i32]
            L.spec_verify_shard_stats_bytes.restype = sz
            L.spec_verify_shard_candidate_bytes.argtypes = [i32]
            L.spec_verify_shard_candidate_bytes.restype = sz
            L.spec_verify_shard_stats.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                  vp, vp, sz, vp]
            L.spec_verify_shard_stats.restype = i32
            L.spec_verify_shard_decide.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                   vp, i32, u64, u64, vp, vp, vp, vp, vp, vp, sz,
                                                   vp]
            L.spec_verify_shard_decide.restype = i32
            L.spec_verify_shard_pick.argtypes = [vp, i32, i32, i32, vp, vp, vp]
            L.spec_verify_shard_pick.restype = i32
            _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        raise SpecVerifyError(rc, lib().spec_verify_last_error().decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return C.c_void_p(stream.cuda_stream)


def _on(device):
    """The C library works on the current CUDA device (its device checks and
    per-device caches ask cudaGetDevice): make the tensors' device current for
    the call."""
    return torch.cuda.device(device)


def workspace_size(B: int, gamma: int, V: int, dtype: int) -> int:
    return int(lib().spec_verify_workspace_size(B, gamma, V, dtype))


def multidraft_workspace_size(B: int, K: int, L: int, V: int, dtype: int) -> int:
    return int(lib().spec_verify_multidraft_workspace_size(B, K, L, V, dtype))


def staging_size(B: int, gamma: int, V: int, dtype: int) -> int:
    return int(lib().spec_verify_host_staging_size(B, gamma, V, dtype))


def _zeroed(nbytes: int, device) -> torch.Tensor:
    # 256-byte alignment is guaranteed by the caching allocator for fresh blocks
    return torch.zeros(max(nbytes, 1), dtype=torch.uint8, device=device)


def spec_verify(target, draft, tokens, temps, *, seed: int = 0, step: int = 0, workspace=None,
                out_accept_len=None, out_tokens=None, out_target_logp=None, out_draft_logp=None,
                with_logprobs: bool = False, stream=None):
    """Verify a batch: target [B, g+1, V], draft [B, g, V] (bf16/fp32), tokens
    [B, g] int32, temps [B] fp32, all on one CUDA device.  Returns
    (accept_len [B], tokens [B, g+1], target_logp, draft_logp)."""
    for t, n in ((target, "target"), (draft, "draft"), (tokens, "tokens"), (temps, "temps")):
        _dev(t, n)
    B, g1, V = target.shape
    g = g1 - 1
    dt = _dt(target)
    if draft.dtype != target.dtype or tuple(draft.shape) != (B, g, V):
        raise ValueError("draft must match target's dtype and be [B, gamma, V]")
    if tokens.dtype != torch.int32 or tuple(tokens.shape) != (B, g):
        raise ValueError("tokens must be int32 [B, gamma]")
    if temps.dtype != torch.float32 or tuple(temps.shape) != (B,):
        raise ValueError("temps must be float32 [B]")
    dev = target.device
    if out_accept_len is None:
        out_accept_len = torch.empty(B, dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, g + 1), dtype=torch.int32, device=dev)
    if with_logprobs and out_target_logp is None:
        out_target_logp = torch.empty((B, g), dtype=torch.float32, device=dev)
    if with_logprobs and out_draft_logp is None:
        out_draft_logp = torch.empty((B, g), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _zeroed(workspace_size(B, g, V, dt), dev)
    with _on(dev):
            _check(lib().spec_verify(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, g, V,
                                 dt, seed, step, _ptr(out_accept_len), _ptr(out_tokens),
                                 _ptr(out_target_logp), _ptr(out_draft_logp), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(),
                                 _stream(dev, stream)))
    return out_accept_len, out_tokens, out_target_logp, out_draft_logp


def spec_verify_multidraft(target, draft, tokens, temps, *, seed: int = 0, step: int = 0,
                           workspace=None, out_accept_len=None, out_tokens=None,
                           out_draft_index=None, stream=None):
    """Multi-draft verification: target [B, L+1, V], draft [B, L, V] shared by
    the K drafts, tokens [B, K, L] int32, temps [B]; or, with a row set per
    draft (the prefix-conditioned use), target [B, K, L+1, V] and draft
    [B, K, L, V].  Returns (accept_len, tokens [B, L+1], draft_index)."""
    for t, n in ((target, "target"), (draft, "draft"), (tokens, "tokens"), (temps, "temps")):
        _dev(t, n)
    per_draft = target.dim() == 4
    if per_draft:
        B, Kt, l1, V = target.shape
    else:
        B, l1, V = target.shape
    L = l1 - 1
    K = tokens.shape[1]
    dt = _dt(target)
    lead = (B, K) if per_draft else (B,)
    if per_draft and Kt != K:
        raise ValueError("per-draft rows: target [B, K, L+1, V] with K = tokens.shape[1]")
    if draft.dtype != target.dtype or tuple(draft.shape) != lead + (L, V):
        raise ValueError("draft must match target's dtype and be [B, L, V] ([B, K, L, V] with "
                         "a row set per draft)")
    if tokens.dtype != torch.int32 or tuple(tokens.shape) != (B, K, L):
        raise ValueError("tokens must be int32 [B, K, L]")
    if temps.dtype != torch.float32 or tuple(temps.shape) != (B,):
        raise ValueError("temps must be float32 [B]")
    dev = target.device
    if out_accept_len is None:
        out_accept_len = torch.empty(B, dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, L + 1), dtype=torch.int32, device=dev)
    if out_draft_index is None:
        out_draft_index = torch.empty(B, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _zeroed(multidraft_workspace_size(B, K, L, V, dt), dev)
    fn = lib().spec_verify_multidraft_rows if per_draft else lib().spec_verify_multidraft
    with _on(dev):
        _check(fn(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, K, L, V, dt, seed,
                  step, _ptr(out_accept_len), _ptr(out_tokens), _ptr(out_draft_index),
                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                  _stream(dev, stream)))
    return out_accept_len, out_tokens, out_draft_index


def spec_verify_host(target, draft, tokens, temps, *, staging, seed: int = 0, step: int = 0,
                     out_accept_len=None, out_tokens=None, stream=None, with_logprobs=False,
                     wait: bool = True):
    """spec_verify on host (preferably pinned) CPU tensors through the C ABI's
    host-buffer entry point; `staging` is a zero-initialised CUDA uint8 tensor
    of at least staging_size(...) bytes.  wait=True returns after the outputs
    have arrived (spec_verify_host); wait=False only enqueues the copies and
    the verification on the stream (spec_verify_host_async): the outputs are
    valid once the stream has reached that point."""
    B, g1, V = target.shape
    g = g1 - 1
    dt = _dt(target)
    for t, n in ((target, "target"), (draft, "draft"), (tokens, "tokens"), (temps, "temps")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor")
    if out_accept_len is None:
        out_accept_len = torch.empty(B, dtype=torch.int32, pin_memory=True)
    if out_tokens is None:
        out_tokens = torch.empty((B, g + 1), dtype=torch.int32, pin_memory=True)
    lp = torch.empty((B, g), dtype=torch.float32, pin_memory=True) if with_logprobs else None
    lq = torch.empty((B, g), dtype=torch.float32, pin_memory=True) if with_logprobs else None
    fn = lib().spec_verify_host if wait else lib().spec_verify_host_async
    with _on(staging.device):
        _check(fn(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, g, V, dt, seed, step,
                  _ptr(out_accept_len), _ptr(out_tokens), _ptr(lp), _ptr(lq), _ptr(staging),
                  staging.numel() * staging.element_size(), _stream(staging.device, stream)))
    return out_accept_len, out_tokens, lp, lq


def spec_verify_noalloc(target, draft, tokens, temps, *, seed: int = 0, step: int = 0,
                        out_accept_len, out_tokens, out_target_logp=None, out_draft_logp=None,
                        stream=None):
    """spec_verify for callers that cannot allocate device memory while they
    verify (memory reserved up front for weights and KV cache, or a decode
    path that must not enter an allocator): the scratch space is a fixed
    array inside the library (``spec_verify_noalloc_max_workspace()`` bytes
    per device), so the call allocates nothing.  Every output tensor must be
    passed in.  The first call on a device sets that array up (make it before
    any stream capture); calls that may overlap on the GPU race."""
    for t, n in ((target, "target"), (draft, "draft"), (tokens, "tokens"), (temps, "temps"),
                 (out_accept_len, "out_accept_len"), (out_tokens, "out_tokens")):
        _dev(t, n)
    B, g1, V = target.shape
    with _on(target.device):
        _check(lib().spec_verify_noalloc(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B,
                                         g1 - 1, V, _dt(target), seed, step,
                                         _ptr(out_accept_len), _ptr(out_tokens),
                                         _ptr(out_target_logp), _ptr(out_draft_logp),
                                         _stream(target.device, stream)))
    return out_accept_len, out_tokens, out_target_logp, out_draft_logp


def spec_verify_noalloc_max_workspace() -> int:
    """Bytes of the fixed scratch array behind spec_verify_noalloc."""
    return int(lib().spec_verify_noalloc_max_workspace())


# ------------------------------------------------------------ vocabulary shards
SHARD_ALIGN = 1024  # shard offsets are multiples of one race group


def vocab_shards(V: int, n: int):
    """[(v0, Vs)] for n ranks over a vocabulary of V: widths rounded up to
    multiples of SHARD_ALIGN (the last shard takes the rest), so no race group
    straddles two ranks.  Ranks past the end of the vocabulary get no shard
    (Vs == 0) and must not call the shard entry points."""
    if V < 1 or n < 1:
        raise ValueError("V and n must be positive")
    w = -(-V // n)
    w = -(-w // SHARD_ALIGN) * SHARD_ALIGN
    out = []
    for r in range(n):
        v0 = min(r * w, V)
        out.append((v0, min(w, V - v0)))
    return out


def shard_stats_bytes(B: int, gamma: int) -> int:
    return int(lib().spec_verify_shard_stats_bytes(B, gamma))


def shard_candidate_bytes(B: int) -> int:
    return int(lib().spec_verify_shard_candidate_bytes(B))


def _shard_inputs(target, draft, tokens, temps):
    for t, n in ((target, "target"), (draft, "draft"), (tokens, "tokens"), (temps, "temps")):
        _dev(t, n)
    B, g1, Vs = target.shape
    g = g1 - 1
    if draft.dtype != target.dtype or tuple(draft.shape) != (B, g, Vs):
        raise ValueError("draft shard must match target's dtype and be [B, gamma, Vs]")
    if tokens.dtype != torch.int32 or tuple(tokens.shape) != (B, g):
        raise ValueError("tokens must be int32 [B, gamma]")
    if temps.dtype != torch.float32 or tuple(temps.shape) != (B,):
        raise ValueError("temps must be float32 [B]")
    return B, g, Vs, _dt(target)


def spec_verify_shard_stats(target, draft, tokens, temps, *, V: int, v0: int, workspace,
                            out_stats=None, stream=None):
    """Call 1 of vocabulary-sharded verification on this rank's shard
    (target [B, g+1, Vs], draft [B, g, Vs] = columns [v0, v0 + Vs) of the
    full rows).  Returns the rank's statistics record (uint8)."""
    B, g, Vs, dt = _shard_inputs(target, draft, tokens, temps)
    dev = target.device
    if out_stats is None:
        out_stats = torch.empty(max(shard_stats_bytes(B, g), 16), dtype=torch.uint8, device=dev)
    with _on(dev):
        _check(lib().spec_verify_shard_stats(
            _ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, g, V, v0, Vs, dt,
            _ptr(out_stats), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(dev, stream)))
    return out_stats


def spec_verify_shard_decide(target, draft, tokens, temps, all_stats, *, V: int, v0: int,
                             nshards: int, workspace, seed: int = 0, step: int = 0,
                             out_accept_len=None, out_tokens=None, with_logprobs: bool = False,
                             out_candidate=None, stream=None):
    """Call 2: the decision from the gathered records of all nshards ranks,
    and this shard's race candidate.  Returns (accept_len, tokens, lp, lq,
    candidate); tokens[b][accept_len[b]] is filled by call 3."""
    B, g, Vs, dt = _shard_inputs(target, draft, tokens, temps)
    _dev(all_stats, "all_stats")
    dev = target.device
    if out_accept_len is None:
        out_accept_len = torch.empty(B, dtype=torch.int32, device=dev)
    if out_tokens is None:
        out_tokens = torch.empty((B, g + 1), dtype=torch.int32, device=dev)
    lp = torch.empty((B, g), dtype=torch.float32, device=dev) if with_logprobs else None
    lq = torch.empty((B, g), dtype=torch.float32, device=dev) if with_logprobs else None
    if out_candidate is None:
        out_candidate = torch.empty(max(shard_candidate_bytes(B), 16), dtype=torch.uint8,
                                    device=dev)
    with _on(dev):
        _check(lib().spec_verify_shard_decide(
            _ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, g, V, v0, Vs, dt,
            _ptr(all_stats), nshards, seed, step, _ptr(out_accept_len), _ptr(out_tokens),
            _ptr(lp), _ptr(lq), _ptr(out_candidate), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(dev, stream)))
    return out_accept_len, out_tokens, lp, lq, out_candidate


def spec_verify_shard_pick(all_candidates, *, nshards: int, out_accept_len, out_tokens,
                           stream=None):
    """Call 3: the drawn token from the gathered candidates of all ranks."""
    for t, n in ((all_candidates, "all_candidates"), (out_accept_len, "out_accept_len"),
                 (out_tokens, "out_tokens")):
        _dev(t, n)
    B, g1 = out_tokens.shape
    dev = out_tokens.device
    with _on(dev):
        _check(lib().spec_verify_shard_pick(_ptr(all_candidates), nshards, B, g1 - 1,
                                            _ptr(out_accept_len), _ptr(out_tokens),
                                            _stream(dev, stream)))
    return out_accept_len, out_tokens


def gather_records(local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of one byte record per rank, concatenated in rank order
    (the exchange between the shard calls)."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    out = torch.empty(n * local.numel(), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(out, local, group=group)
    return out


def spec_verify_vocab_sharded(target, draft, tokens, temps, *, V: int, v0: int, seed: int = 0,
                              step: int = 0, group=None, workspace=None,
                              with_logprobs: bool = False, exchange=gather_records):
    """The three shard calls with the two exchanges between them, on this
    rank of `group` (every rank of the group calls it with its own shard).
    Returns (accept_len, tokens, lp, lq), the same on every rank."""
    import torch.distributed as dist
    n = dist.get_world_size(group)
    B, g, Vs, dt = _shard_inputs(target, draft, tokens, temps)
    if workspace is None:
        workspace = _zeroed(workspace_size(B, g, Vs, dt), target.device)
    stats = spec_verify_shard_stats(target, draft, tokens, temps, V=V, v0=v0,
                                    workspace=workspace)
    all_stats = exchange(stats, group)
    acc, tok, lp, lq, cand = spec_verify_shard_decide(
        target, draft, tokens, temps, all_stats, V=V, v0=v0, nshards=n, workspace=workspace,
        seed=seed, step=step, with_logprobs=with_logprobs)
    spec_verify_shard_pick(exchange(cand, group), nshards=n, out_accept_len=acc,
                           out_tokens=tok)
    return acc, tok, lp, lq


class Verifier:
    """Owns a zero-initialised workspace sized for the largest shape seen."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self._ws = None

    def _workspace(self, nbytes):
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = _zeroed(nbytes, self.device)
        return self._ws

    def verify(self, target, draft, tokens, temps, **kw):
        B, g1, V = target.shape
        ws = self._workspace(workspace_size(B, g1 - 1, V, _dt(target)))
        return spec_verify(target, draft, tokens, temps, workspace=ws, **kw)

    def verify_multidraft(self, target, draft, tokens, temps, **kw):
        B, l1, V = target.shape[0], target.shape[-2], target.shape[-1]
        ws = self._workspace(multidraft_workspace_size(B, tokens.shape[1], l1 - 1, V,
                                                       _dt(target)))
        return spec_verify_multidraft(target, draft, tokens, temps, workspace=ws, **kw)


class Bandit:
    """Online draft selection (include/sv_bandit.h): K arms, policy "ucb1" or
    "thompson".  select() gives the arm (draft model) for the next step;
    update(arm, reward) or update_from_accept(arm, accept_len, gamma) records
    the outcome.  Host-side by design: accept_len is read from the host (a
    device tensor is copied back, B int32 values)."""

    POLICIES = {"ucb1": 0, "thompson": 1}

    def __init__(self, K: int, policy: str = "ucb1", seed: int = 0):
        if policy not in self.POLICIES:
            raise ValueError(f"policy must be one of {sorted(self.POLICIES)}")
        self.K = K
        self._h = lib().sv_bandit_create(K, self.POLICIES[policy], seed)
        if not self._h:
            raise SpecVerifyError(1, lib().spec_verify_last_error().decode())

    def select(self) -> int:
        arm = C.c_int(-1)
        _check(lib().sv_bandit_select(self._h, C.byref(arm)))
        return arm.value

    def update(self, arm: int, reward: float) -> None:
        _check(lib().sv_bandit_update(self._h, arm, float(reward)))

    def update_from_accept(self, arm: int, accept_len, gamma: int) -> None:
        a = torch.as_tensor(accept_len).to("cpu", torch.int32).contiguous()
        _check(lib().sv_bandit_update_accept(self._h, arm, a.data_ptr() if a.numel() else None,
                                             a.numel(), gamma))

    def stats(self):
        pulls = torch.zeros(self.K, dtype=torch.int64)
        sums = torch.zeros(self.K, dtype=torch.float64)
        _check(lib().sv_bandit_stats(self._h, pulls.data_ptr(), sums.data_ptr()))
        return pulls, sums

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().sv_bandit_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: the library may already be gone
            pass
