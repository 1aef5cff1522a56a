"""The oracle's tie rule for the correction draw, pinned against the error
model it states (CPU).

The rule: a draw is logged as a Gumbel near-tie when another candidate's
score could overtake the winner's once every probability carries the
relative error eta = 2e-6 + 2e-7 |ln prob| of an fp32 evaluation.  A
residual weight p - q of two nearly equal probabilities amplifies that error
by (p + q) / (p - q), so the band widens there.

Pin: on near-equality residual draws (the regime where the fixed band alone
is too narrow), perturb every p and q at random within the stated error and
redo the Gumbel-max by brute force (numpy, the pages' definition: argmax of
ln max(p - q, 0) + G with the keyed noise).  Whenever the perturbed winner
differs from the oracle's token, the oracle must have logged the tie; and
the unperturbed brute force must reproduce the oracle's token.  Control: the
fixed band alone (gap < 1e-4) misses some of those flips.
"""
from __future__ import annotations

import numpy as np

import oracle

ETA0, ETA1, BAND = 2e-6, 2e-7, 1e-4


def _scores_noise(V, seed, step, b, pos):
    lnE = np.empty(V)
    for v in range(V):
        x = oracle.stream_word(seed, step, 2, b, 0, pos, v >> 2, v & 3)
        U = oracle.u01_gumbel(x)
        lnE[v] = np.log(-np.log1p(-(1.0 - U)))
    return -lnE  # G_v = -ln E_v


def _near_equal_case(rng, V):
    """One sequence, gamma = 1: the draft row is the target row plus N(0,
    1e-4) noise, except that the draft token -- a low-probability entry -- is
    boosted by +2 in the draft row (rejected with probability ~0.86), so the
    residual max(p - q, 0) is a difference of nearly equal probabilities."""
    tgt = rng.normal(0.0, 2.0, (1, 2, V)).astype(np.float32)
    drf = (tgt[:, :1] + rng.normal(0.0, 1e-4, (1, 1, V))).astype(np.float32)
    x = int(np.argmin(tgt[0, 0]))
    drf[0, 0, x] += 2.0
    return tgt, drf, np.array([[x]], dtype=np.int32), np.array([1.0], dtype=np.float32)


def test_tie_rule_covers_fp32_evaluation_error():
    rng = np.random.default_rng(20)
    flips = flips_logged = flips_fixed_band = draws = 0
    for case in range(200):
        V = 64
        tgt, drf, tok, tm = _near_equal_case(rng, V)
        seed, step = 3, case
        r = oracle.verify(tgt, drf, tok, tm, seed=seed, step=step)
        if r["accept_len"][0] != 0:
            continue  # accepted: no residual draw
        draws += 1
        y, tie = int(r["tokens"][0, 0]), int(r["tie"][0])
        lp = oracle.row_logprobs(tgt[0, 0], 1.0)
        lq = oracle.row_logprobs(drf[0, 0], 1.0)
        G = _scores_noise(V, seed, step, 0, 0)
        p, q = np.exp(lp), np.exp(lq)

        def winner(pp, qq):
            w = np.maximum(pp - qq, 0.0)
            with np.errstate(divide="ignore"):
                s = np.where(w > 0, np.log(w), -np.inf) + G
            return int(np.argmax(s)), s

        y0, s0 = winner(p, q)
        assert y0 == y  # brute force reproduces the oracle's draw
        top = np.sort(s0[np.isfinite(s0)])[::-1]
        gap = top[0] - top[1] if top.size > 1 else np.inf
        for _ in range(40):
            ep = (ETA0 + ETA1 * np.abs(lp)) * rng.uniform(-1.0, 1.0, V)
            eq = (ETA0 + ETA1 * np.abs(lq)) * rng.uniform(-1.0, 1.0, V)
            y1, _ = winner(p * (1.0 + ep), q * (1.0 + eq))
            if y1 != y:
                flips += 1
                flips_logged += bool(tie & oracle.TIE_GUMBEL)
                flips_fixed_band += gap < BAND
    print(f"draws {draws} flips {flips} logged {flips_logged} fixed-band {flips_fixed_band}")
    assert draws >= 120
    assert flips > 0  # the regime does produce fp32-sized flips
    assert flips_logged == flips  # every one of them is logged by the rule
    assert flips_fixed_band < flips  # control: the fixed band alone misses some


def test_tie_rule_is_the_fixed_band_for_well_conditioned_draws():
    """Bonus draws (w = p) and residuals of clearly different rows: the band
    reduces to the fixed 1e-4 (a flagged draw has a top-2 gap below ~1e-4)."""
    rng = np.random.default_rng(21)
    flagged = 0
    for case in range(40):
        V = 2000
        tgt = rng.normal(0.0, 2.0, (4, 2, V)).astype(np.float32)
        drf = (tgt[:, :1] + rng.normal(0.0, 1.0, (4, 1, V))).astype(np.float32)
        tok = rng.integers(0, V, (4, 1)).astype(np.int32)
        tm = np.ones(4, dtype=np.float32)
        r = oracle.verify(tgt, drf, tok, tm, seed=1, step=case)
        for b in range(4):
            if not r["tie"][b] & oracle.TIE_GUMBEL:
                continue
            flagged += 1
            j = int(r["accept_len"][b])
            lp = oracle.row_logprobs(tgt[b, j], 1.0)
            if j == 0:
                lq = oracle.row_logprobs(drf[b, 0], 1.0)
                lw, _ = oracle.residual_logw(lp, lq)
            else:
                lw = lp
            _, gap = oracle.group_race(lw, 1, case, 2, b, j)
            assert gap < 1.2e-4
    assert flagged <= 3  # about 1e-4 per draw over 160 draws


def _group_noise(ng, seed, step, b, pos):
    lnE = np.empty(ng)
    for g in range(ng):
        U = oracle.u01_gumbel(oracle.stream_word(seed, step, oracle.TAG_GROUP, b, 0, pos, g, 0))
        lnE[g] = np.log(-np.log1p(-(1.0 - U)))
    return -lnE


def test_group_tie_rule_covers_fp32_evaluation_error():
    """The same pin for the group level of the two-level race: rows spanning
    three groups of RACE_GROUP entries, residuals of nearly equal rows (so
    each group's weight is a sum of ill-conditioned differences).  Brute
    force (numpy): group weights W_g = sum max(p - q, 0) over the group, the
    group maximising ln W_g + G_g with the group noise, then the entry
    maximising ln w_v + G_v within it.  Every perturbed flip must be logged."""
    rng = np.random.default_rng(22)
    G = oracle.RACE_GROUP
    flips = flips_logged = draws = group_flips = flips_fixed_band = logged = 0
    for case in range(100):
        V = 2 * G + 700
        ng = (V + G - 1) // G
        tgt = rng.normal(0.0, 2.0, (1, 2, V)).astype(np.float32)
        sigma = 10.0 ** rng.uniform(-4.5, -2.0)  # from ill- to well-conditioned residuals
        drf = (tgt[:, :1] + rng.normal(0.0, sigma, (1, 1, V))).astype(np.float32)
        x = int(np.argmin(tgt[0, 0]))
        drf[0, 0, x] += 2.0
        tok = np.array([[x]], dtype=np.int32)
        tm = np.array([1.0], dtype=np.float32)
        seed, step = 5, case
        r = oracle.verify(tgt, drf, tok, tm, seed=seed, step=step)
        if r["accept_len"][0] != 0:
            continue
        draws += 1
        y, tie = int(r["tokens"][0, 0]), int(r["tie"][0])
        lp = oracle.row_logprobs(tgt[0, 0], 1.0)
        lq = oracle.row_logprobs(drf[0, 0], 1.0)
        Ge = _scores_noise(V, seed, step, 0, 0)
        Gg = _group_noise(ng, seed, step, 0, 0)
        p, q = np.exp(lp), np.exp(lq)

        def winner(pp, qq):
            w = np.maximum(pp - qq, 0.0)
            W = np.array([w[g * G:(g + 1) * G].sum() for g in range(ng)])
            with np.errstate(divide="ignore"):
                sg = np.where(W > 0, np.log(W), -np.inf) + Gg
                g = int(np.argmax(sg))
                se = np.where(w > 0, np.log(w), -np.inf) + Ge
            lo, hi = g * G, min(V, (g + 1) * G)
            return lo + int(np.argmax(se[lo:hi])), g

        y0, g0 = winner(p, q)
        assert y0 == y  # brute force reproduces the oracle's draw
        lw, _ = oracle.residual_logw(lp, lq)
        _, gap = oracle.group_race(lw, seed, step, oracle.TAG_GUMBEL, 0, 0)
        logged += bool(tie & oracle.TIE_GUMBEL)
        for _ in range(20):
            # errors of one sign per group (p up and q down, or the reverse):
            # the direction that moves a group sum the most
            sg = np.repeat(rng.choice([-1.0, 1.0], ng), G)[:V]
            ep = (ETA0 + ETA1 * np.abs(lp)) * rng.uniform(0.0, 1.0, V) * sg
            eq = -(ETA0 + ETA1 * np.abs(lq)) * rng.uniform(0.0, 1.0, V) * sg
            y1, g1 = winner(p * (1.0 + ep), q * (1.0 + eq))
            if y1 != y:
                flips += 1
                group_flips += g1 != g0
                flips_logged += bool(tie & oracle.TIE_GUMBEL)
                flips_fixed_band += gap < BAND
    print(f"draws {draws} (logged {logged}) flips {flips} (group {group_flips}) "
          f"logged {flips_logged} fixed-band {flips_fixed_band}")
    assert draws >= 30
    assert group_flips > 0  # the regime does produce group-level flips
    assert flips_logged == flips  # every one of them is logged by the rule
    assert flips_fixed_band < flips  # control: the fixed band alone misses some
    assert logged < draws  # the rule does not log every draw
