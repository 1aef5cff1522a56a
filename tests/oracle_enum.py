"""Exact enumeration of the oracle's output law.

The oracle draws all randomness through two primitives, a Bernoulli(h) coin
and a categorical draw from log-weights.  Replacing them with a scripted
source and walking every branch (an odometer over the branch choices) gives
the exact probability of every output for fixed inputs; summing over all draft
tuples weighted by their draft probabilities gives the law of the emitted
tokens.  Nothing here restates the verification rule: the oracle's own control
flow, acceptance probabilities and residuals decide the branches and their
weights.
"""
from __future__ import annotations

import itertools

import numpy as np

import oracle


class Script:
    def __init__(self):
        self.script: list[int] = []
        self.trace: list[np.ndarray] = []  # per decision: option probabilities

    def _take(self, probs: np.ndarray) -> int:
        i = len(self.trace)
        self.trace.append(probs)
        if i < len(self.script):
            return self.script[i]
        c = int(np.flatnonzero(probs > 0)[0]) if np.any(probs > 0) else 0
        self.script.append(c)
        return c

    def coin(self, h, tag, b, k, pos):
        h = min(max(float(h), 0.0), 1.0)
        return self._take(np.array([h, 1.0 - h])) == 0

    def categorical(self, logw, tag, b, pos):
        w = np.where(np.isfinite(logw), logw, -np.inf)
        m = np.max(w)
        p = np.exp(w - m)
        p /= p.sum()
        return self._take(p)

    def weight(self) -> float:
        wt = 1.0
        for c, p in zip(self.script, self.trace):
            wt *= float(p[c])
        return wt

    def advance(self) -> bool:
        self.script = self.script[: len(self.trace)]
        i = len(self.trace) - 1
        while i >= 0:
            p = self.trace[i]
            c = self.script[i] + 1
            while c < len(p) and p[c] == 0:
                c += 1
            if c < len(p):
                self.script[i] = c
                del self.script[i + 1:]
                return True
            i -= 1
        return False


def leaves(run_once, script_cls=None):
    """Yield (weight, result) for every branch of run_once(rng)."""
    s = (script_cls or Script)()
    rng = oracle.CallbackRng(s.coin, s.categorical)
    while True:
        s.trace = []
        res = run_once(rng)
        yield s.weight(), res
        if not s.advance():
            break


def row_probs(rows: np.ndarray, T: float) -> np.ndarray:
    """Softmax of each row as the oracle defines it (its log-softmax, exp'd)."""
    return np.stack([np.exp(oracle.row_logprobs(r, T)) for r in rows])


def single_draft_law(target, draft, T, script_cls=None):
    """Exact law of (accept_len, emitted tokens) for one sequence.

    target [gamma+1, V], draft [gamma, V].  Returns a dict mapping
    (accept_len, tokens tuple) -> probability, summed over every draft tuple
    x ~ prod_i Q_i and every branch of the oracle.
    """
    g1, V = target.shape
    gamma = g1 - 1
    Q = row_probs(draft, T)
    temps = np.array([T], dtype=np.float32)
    law: dict = {}
    for x in itertools.product(range(V), repeat=gamma):
        wx = float(np.prod([Q[i, x[i]] for i in range(gamma)]))
        if wx == 0.0:
            continue
        toks = np.array([x], dtype=np.int32)

        def run(rng):
            r = oracle.verify(target[None], draft[None], toks, temps, rng=rng,
                              with_logprobs=False)
            j = int(r["accept_len"][0])
            return j, tuple(int(t) for t in r["tokens"][0, : j + 1])

        for w, key in leaves(run, script_cls):
            law[key] = law.get(key, 0.0) + wx * w
    return law


def multidraft_law(target, draft, K, T):
    """Exact law of (tau, emitted tokens) for one sequence of the multi-draft
    verifier with K i.i.d. drafts, each x_k ~ prod_i Q_i."""
    l1, V = target.shape
    L = l1 - 1
    Q = row_probs(draft, T)
    temps = np.array([T], dtype=np.float32)
    law: dict = {}
    blocks = list(itertools.product(range(V), repeat=L))
    pblock = [float(np.prod([Q[i, blk[i]] for i in range(L)])) for blk in blocks]
    for combo in itertools.product(range(len(blocks)), repeat=K):
        wx = float(np.prod([pblock[c] for c in combo]))
        if wx == 0.0:
            continue
        toks = np.array([[blocks[c] for c in combo]], dtype=np.int32)

        def run(rng):
            r = oracle.verify_multidraft(target[None], draft[None], toks, temps, rng=rng)
            t = int(r["accept_len"][0])
            return t, tuple(int(v) for v in r["tokens"][0, : t + 1])

        for w, key in leaves(run):
            law[key] = law.get(key, 0.0) + wx * w
    return law


def extend_to_full(law, P):
    """Complete every emitted prefix with target draws P_m for the later
    positions (the target law is position-wise here), giving a law over
    V^(n_pos)."""
    n_pos, V = P.shape
    full = np.zeros((V,) * n_pos)
    for (j, toks), w in law.items():
        rest = n_pos - len(toks)
        if rest == 0:
            full[toks] += w
            continue
        tail = P[len(toks)]
        for m in range(len(toks) + 1, n_pos):
            tail = np.multiply.outer(tail, P[m])
        full[toks] += w * tail
    return full


def product_law(P):
    out = P[0]
    for m in range(1, P.shape[0]):
        out = np.multiply.outer(out, P[m])
    return out


# ---------------------------------------------------- prefix-conditioned model
def prefix_model(V: int, L: int, seed: int):
    """A small autoregressive target / draft pair: a logit row for every
    prefix (target rows for prefixes of length 0..L, draft rows for 0..L-1),
    the draft a noisy copy of the target."""
    rng = np.random.default_rng(seed)
    tctx, dctx = {}, {}
    for n in range(L + 1):
        for pre in itertools.product(range(V), repeat=n):
            tctx[pre] = rng.normal(0.0, 1.5, V).astype(np.float32)
            if n < L:
                dctx[pre] = (tctx[pre] + rng.normal(0.0, 1.0, V)).astype(np.float32)
    return tctx, dctx


def per_draft_rows(tctx, dctx, drafts, L):
    """Per-draft rows for drafts x_k: target row (k, i) = tctx[x_k[:i]],
    draft row (k, i) = dctx[x_k[:i]]."""
    tg = np.stack([np.stack([tctx[tuple(x[:i])] for i in range(L + 1)]) for x in drafts])
    dr = np.stack([np.stack([dctx[tuple(x[:i])] for i in range(L)]) for x in drafts])
    return tg, dr


def multidraft_law_prefix_model(tctx, dctx, V, L, K, T, rows=per_draft_rows):
    """Exact law of (tau, emitted tokens) with K i.i.d. drafts from the
    prefix-conditioned draft model, verified with per-draft rows."""
    q = {pre: np.exp(oracle.row_logprobs(r, T)) for pre, r in dctx.items()}
    temps = np.array([T], dtype=np.float32)
    blocks = list(itertools.product(range(V), repeat=L))
    pblock = [float(np.prod([q[blk[:i]][blk[i]] for i in range(L)])) for blk in blocks]
    law: dict = {}
    for combo in itertools.product(range(len(blocks)), repeat=K):
        wx = float(np.prod([pblock[c] for c in combo]))
        if wx == 0.0:
            continue
        drafts = [blocks[c] for c in combo]
        tg, dr = rows(tctx, dctx, drafts, L)
        toks = np.array([drafts], dtype=np.int32)

        def run(rng):
            r = oracle.verify_multidraft(tg[None], dr[None], toks, temps, rng=rng)
            t = int(r["accept_len"][0])
            return t, tuple(int(v) for v in r["tokens"][0, : t + 1])

        for w, key in leaves(run):
            law[key] = law.get(key, 0.0) + wx * w
    return law


def prefix_target_law(tctx, V, L, T):
    """Law of the target model over V^(L+1): prod_m P(seq[:m])(seq[m])."""
    p = {pre: np.exp(oracle.row_logprobs(r, T)) for pre, r in tctx.items()}
    full = np.zeros((V,) * (L + 1))
    for seq in itertools.product(range(V), repeat=L + 1):
        full[seq] = float(np.prod([p[seq[:m]][seq[m]] for m in range(L + 1)]))
    return full, p


def extend_prefix_law(law, p, V, L):
    """Complete every emitted prefix with target draws from the
    prefix-conditioned target for the later positions."""
    full = np.zeros((V,) * (L + 1))
    for (_, toks), w in law.items():
        n = len(toks)
        for rest in itertools.product(range(V), repeat=L + 1 - n):
            seq = tuple(toks) + rest
            full[seq] += w * float(np.prod([p[seq[:m]][seq[m]] for m in range(n, L + 1)]))
    return full
