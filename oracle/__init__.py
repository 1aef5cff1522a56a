"""CPU oracle for batched speculative-sampling verification (ctypes binding).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the CUDA library and its Python binding) never imports, links or calls
it, and it never imports the product.

The arithmetic lives in ``sv_oracle.c`` (plain single-threaded C, fp64 after
the fp32 temperature scaling); this module only marshals numpy arrays.  The
harness may run disjoint batch ranges on several host threads (ctypes drops
the GIL during the foreign call); each call is still the single-threaded
definition.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsvoracle.so")

F32, BF16 = 0, 1
TAG_ACCEPT, TAG_GUMBEL, TAG_MD_ETA, TAG_MD_GUMBEL = 1, 2, 3, 4
TAG_GROUP = 7
RACE_GROUP = 1024  # vocabulary entries per group of the single-draft two-level race
TIE_BERNOULLI, TIE_GUMBEL = 1, 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "sv_oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = [
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm",
        ]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


COIN_FN = C.CFUNCTYPE(C.c_int, C.c_void_p, C.c_double, C.c_uint32, C.c_uint32,
                      C.c_uint32, C.c_uint32, C.POINTER(C.c_double))
CAT_FN = C.CFUNCTYPE(C.c_int64, C.c_void_p, C.POINTER(C.c_double), C.c_int64,
                     C.c_uint32, C.c_uint32, C.c_uint32, C.POINTER(C.c_double))


class Rng(C.Structure):
    _fields_ = [("ctx", C.c_void_p), ("coin", COIN_FN), ("categorical", CAT_FN)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            vp, i64, u64, u32 = C.c_void_p, C.c_int64, C.c_uint64, C.c_uint32
            L.svo_philox4x32_10.argtypes = [vp, vp, vp]
            L.svo_u01_accept.argtypes = [u32]
            L.svo_u01_accept.restype = C.c_double
            L.svo_u01_gumbel.argtypes = [u32]
            L.svo_u01_gumbel.restype = C.c_double
            L.svo_stream_word.argtypes = [u64, u64, u32, u32, u32, u32, u32, u32]
            L.svo_stream_word.restype = u32
            L.svo_bf16_to_f32.argtypes = [C.c_uint16]
            L.svo_bf16_to_f32.restype = C.c_float
            L.svo_row_logprobs.argtypes = [vp, i64, C.c_int, C.c_float, vp]
            L.svo_row_logprobs.restype = C.c_int
            L.svo_row_argmax.argtypes = [vp, i64, C.c_int]
            L.svo_row_argmax.restype = i64
            L.svo_residual_logw.argtypes = [vp, vp, i64, vp]
            L.svo_residual_logw.restype = i64
            L.svo_gumbel_argmax.argtypes = [vp, i64, u64, u64, u32, u32, u32, vp]
            L.svo_gumbel_argmax.restype = i64
            L.svo_group_race.argtypes = [vp, i64, u64, u64, u32, u32, u32, vp]
            L.svo_group_race.restype = i64
            L.svo_verify.argtypes = [vp, vp, vp, vp, i64, C.c_int, i64, C.c_int, u64, u64,
                                     i64, i64, vp, vp, vp, vp, vp, C.POINTER(Rng)]
            L.svo_verify.restype = C.c_int
            L.svo_verify_multidraft.argtypes = [vp, vp, vp, vp, i64, C.c_int, C.c_int, i64,
                                                C.c_int, u64, u64, i64, i64, vp, vp, vp, vp,
                                                C.POINTER(Rng)]
            L.svo_verify_multidraft.restype = C.c_int
            L.svo_verify_multidraft_rows.argtypes = [vp, vp, vp, vp, i64, C.c_int, C.c_int, i64,
                                                     C.c_int, C.c_int, u64, u64, i64, i64, vp, vp,
                                                     vp, vp, C.POINTER(Rng)]
            L.svo_verify_multidraft_rows.restype = C.c_int
            L.svo_bandit_uniform.argtypes = [u64, u32, u32, u32, u32, C.c_int]
            L.svo_bandit_uniform.restype = C.c_double
            L.svo_gamma_sample.argtypes = [C.c_double, u64, u32, u32]
            L.svo_gamma_sample.restype = C.c_double
            L.svo_beta_sample.argtypes = [C.c_double, C.c_double, u64, u32, u32]
            L.svo_beta_sample.restype = C.c_double
            L.svo_ucb1_select.argtypes = [C.c_int, vp, vp]
            L.svo_ucb1_select.restype = C.c_int
            L.svo_thompson_select.argtypes = [C.c_int, vp, vp, u64, u32, vp]
            L.svo_thompson_select.restype = C.c_int
            L.svo_thompson_trial.argtypes = [C.c_double, u64, u32, u32]
            L.svo_thompson_trial.restype = C.c_int
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _dtype_code(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:  # raw bf16 bit patterns
        return BF16
    raise TypeError("logits must be float32 or uint16 (bf16 bits)")


# ---------------------------------------------------------------- primitives
def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().svo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def stream_word(seed, step, tag, b, k, pos, c0, w) -> int:
    return int(lib().svo_stream_word(seed, step, tag, b, k, pos, c0, w))


def u01_accept(x: int) -> float:
    return float(lib().svo_u01_accept(x))


def u01_gumbel(x: int) -> float:
    return float(lib().svo_u01_gumbel(x))


def bf16_to_f32(bits: int) -> float:
    return float(lib().svo_bf16_to_f32(bits))


def row_logprobs(row: np.ndarray, T: float):
    row = np.ascontiguousarray(row)
    out = np.empty(row.shape[-1], dtype=np.float64)
    rc = lib().svo_row_logprobs(_ptr(row), row.shape[-1], _dtype_code(row), T, _ptr(out))
    return None if rc != 0 else out


def row_argmax(row: np.ndarray) -> int:
    row = np.ascontiguousarray(row)
    return int(lib().svo_row_argmax(_ptr(row), row.shape[-1], _dtype_code(row)))


def residual_logw(lp: np.ndarray, lq: np.ndarray):
    lp = np.ascontiguousarray(lp, dtype=np.float64)
    lq = np.ascontiguousarray(lq, dtype=np.float64)
    out = np.empty_like(lp)
    n = lib().svo_residual_logw(_ptr(lp), _ptr(lq), lp.size, _ptr(out))
    return out, int(n)


def gumbel_argmax(logw: np.ndarray, seed, step, tag, b, pos):
    logw = np.ascontiguousarray(logw, dtype=np.float64)
    gap = np.zeros(1, dtype=np.float64)
    y = lib().svo_gumbel_argmax(_ptr(logw), logw.size, seed, step, tag, b, pos, _ptr(gap))
    return int(y), float(gap[0])


def group_race(logw: np.ndarray, seed, step, tag, b, pos):
    """The single-draft draw: two-level exponential race (groups of RACE_GROUP)."""
    logw = np.ascontiguousarray(logw, dtype=np.float64)
    gap = np.zeros(1, dtype=np.float64)
    y = lib().svo_group_race(_ptr(logw), logw.size, seed, step, tag, b, pos, _ptr(gap))
    return int(y), float(gap[0])


# --------------------------------------------------------------- randomness
class CallbackRng:
    """Wrap Python callables as the oracle's randomness source.

    coin(h, tag, b, k, pos) -> bool; categorical(logw: np.ndarray, tag, b, pos) -> int.
    """

    def __init__(self, coin, categorical):
        def _coin(_ctx, h, tag, b, k, pos, _gap):
            return 1 if coin(h, tag, b, k, pos) else 0

        def _cat(_ctx, logw_p, V, tag, b, pos, _gap):
            logw = np.ctypeslib.as_array(logw_p, shape=(V,)).copy()
            return int(categorical(logw, tag, b, pos))

        self._c = COIN_FN(_coin)
        self._k = CAT_FN(_cat)
        self.struct = Rng(None, self._c, self._k)


# ------------------------------------------------------------- verification
def _ranges(B: int, threads: int):
    threads = max(1, min(threads, B))
    step = (B + threads - 1) // threads
    return [(s, min(B, s + step)) for s in range(0, B, step)]


def verify(target, draft, tokens, temps, *, seed=0, step=0, rng=None, threads=1,
           with_logprobs=True):
    """Single-draft verification of a batch.

    target [B, gamma+1, V], draft [B, gamma, V] as float32 or uint16 (bf16
    bits); tokens [B, gamma] int32; temps [B] float32.  Returns a dict with
    accept_len [B], tokens [B, gamma+1], lp/lq [B, gamma] (fp64), tie [B].
    """
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    temps = np.ascontiguousarray(temps, dtype=np.float32)
    B, g1, V = target.shape
    gamma = g1 - 1
    assert draft.shape == (B, gamma, V) and tokens.shape == (B, gamma) and temps.shape == (B,)
    dt = _dtype_code(target)
    assert _dtype_code(draft) == dt
    acc = np.empty(B, dtype=np.int32)
    tok = np.empty((B, gamma + 1), dtype=np.int32)
    lp = np.empty((B, gamma), dtype=np.float64) if with_logprobs else None
    lq = np.empty((B, gamma), dtype=np.float64) if with_logprobs else None
    tie = np.empty(B, dtype=np.uint8)
    rng_p = C.byref(rng.struct) if rng is not None else None
    L = lib()

    def run(r):
        rc = L.svo_verify(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps), B, gamma, V, dt,
                          seed, step, r[0], r[1], _ptr(acc), _ptr(tok), _ptr(lp), _ptr(lq),
                          _ptr(tie), rng_p)
        if rc != 0:
            raise ValueError("svo_verify rejected its arguments")

    if rng is not None or threads <= 1:
        run((0, B))
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, _ranges(B, threads)))
    return {"accept_len": acc, "tokens": tok, "lp": lp, "lq": lq, "tie": tie}


def verify_multidraft(target, draft, tokens, temps, *, seed=0, step=0, rng=None, threads=1):
    """Multi-draft verification.  target [B, L+1, V] and draft [B, L, V] shared
    by the K drafts, or per-draft rows target [B, K, L+1, V] and draft
    [B, K, L, V] (row (k, i) conditioned on draft k's own prefix); tokens
    [B, K, L].  Returns accept_len [B], tokens [B, L+1], draft_index [B], tie [B]."""
    target = np.ascontiguousarray(target)
    draft = np.ascontiguousarray(draft)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    temps = np.ascontiguousarray(temps, dtype=np.float32)
    per_draft = target.ndim == 4
    B, K = tokens.shape[0], tokens.shape[1]
    l1, V = target.shape[-2], target.shape[-1]
    L_ = l1 - 1
    lead = (B, K) if per_draft else (B,)
    assert target.shape == lead + (L_ + 1, V) and draft.shape == lead + (L_, V)
    assert tokens.shape == (B, K, L_) and temps.shape == (B,)
    dt = _dtype_code(target)
    assert _dtype_code(draft) == dt
    acc = np.empty(B, dtype=np.int32)
    tok = np.empty((B, L_ + 1), dtype=np.int32)
    didx = np.empty(B, dtype=np.int32)
    tie = np.empty(B, dtype=np.uint8)
    rng_p = C.byref(rng.struct) if rng is not None else None
    Lb = lib()

    def run(r):
        rc = Lb.svo_verify_multidraft_rows(_ptr(target), _ptr(draft), _ptr(tokens), _ptr(temps),
                                           B, K, L_, V, dt, int(per_draft), seed, step, r[0],
                                           r[1], _ptr(acc), _ptr(tok), _ptr(didx), _ptr(tie),
                                           rng_p)
        if rc != 0:
            raise ValueError("svo_verify_multidraft_rows rejected its arguments")

    if rng is not None or threads <= 1:
        run((0, B))
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(run, _ranges(B, threads)))
    return {"accept_len": acc, "tokens": tok, "draft_index": didx, "tie": tie}


# ------------------------------------------------------- draft selection bandit
def gamma_sample(alpha: float, seed: int, round_: int, slot: int) -> float:
    return lib().svo_gamma_sample(alpha, seed, round_, slot)


def beta_sample(a: float, b: float, seed: int, round_: int, arm: int) -> float:
    return lib().svo_beta_sample(a, b, seed, round_, arm)


def bandit_uniform(seed: int, c0: int, round_: int, slot: int, tag: int, half: int = 0) -> float:
    return lib().svo_bandit_uniform(seed, c0, round_, slot, tag, half)


def ucb1_select(pulls, reward_sum) -> int:
    n = np.ascontiguousarray(pulls, dtype=np.int64)
    s = np.ascontiguousarray(reward_sum, dtype=np.float64)
    return int(lib().svo_ucb1_select(len(n), _ptr(n), _ptr(s)))


def thompson_select(succ, fail, seed: int, round_: int):
    S = np.ascontiguousarray(succ, dtype=np.int64)
    F = np.ascontiguousarray(fail, dtype=np.int64)
    theta = np.empty(len(S), dtype=np.float64)
    arm = int(lib().svo_thompson_select(len(S), _ptr(S), _ptr(F), seed, round_, _ptr(theta)))
    return arm, theta


def thompson_trial(reward: float, seed: int, round_: int, arm: int) -> bool:
    return bool(lib().svo_thompson_trial(reward, seed, round_, arm))


class BanditOracle:
    """The selector's state machine, step by step: select() at select round
    t_s, update(arm, reward) at update round t_u (both count from 0)."""

    def __init__(self, K: int, policy: str = "ucb1", seed: int = 0):
        self.K, self.policy, self.seed = K, policy, seed
        self.pulls = np.zeros(K, np.int64)
        self.sums = np.zeros(K, np.float64)
        self.succ = np.zeros(K, np.int64)
        self.fail = np.zeros(K, np.int64)
        self.t_s = self.t_u = 0

    def select(self) -> int:
        if self.policy == "ucb1":
            arm = ucb1_select(self.pulls, self.sums)
        else:
            arm, _ = thompson_select(self.succ, self.fail, self.seed, self.t_s)
        self.t_s += 1
        return arm

    def update(self, arm: int, reward: float) -> None:
        self.pulls[arm] += 1
        self.sums[arm] += reward
        if self.policy != "ucb1":
            if thompson_trial(reward, self.seed, self.t_u, arm):
                self.succ[arm] += 1
            else:
                self.fail[arm] += 1
        self.t_u += 1
