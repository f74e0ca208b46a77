"""Exact enumeration of the law of the tokens a verify step emits, at tiny V and K.

Shared by the oracle's pins (tests/test_oracle_pins.py) and the same check on the CUDA path
(tests/test_gpu_lossless.py). The rule is exactly lossless when the joint law of the K+1
emitted tokens equals p_1 x ... x p_{K+1} (dspark-mlx wheel, adapter.py docstring, "lossless
accept policy"; DeepSeek-V4-Flash DSpark drafter card, "lossless by construction").

Method. Rows have rational probabilities whose denominators divide ``denom``. Every ratio
p/q and every normalised CDF point of any residual then lies in the Farey sequence
F_denom, so a verify step's output is constant on each interval between consecutive members
and the interval's midpoint decides it. Each uniform coordinate is swept over those
intervals (weight: the interval's length), each draft tuple is weighted by its draft-law
probability, and tokens the cycle does not emit are continued with p_{n+2}..p_{K+1}, as a
prefix-independent target produces them. All weights are exact rationals.
"""

import itertools
from fractions import Fraction

import numpy as np

from oracle import accept_ref as ora


def logits_of(probs, T=1.0):
    """Logits whose softmax at temperature T is exactly the given probabilities (0 -> -inf)."""
    p = np.asarray([float(x) for x in probs])
    with np.errstate(divide="ignore"):
        return np.log(p) * T


def farey(n):
    """All fractions a/b in [0, 1] with b <= n, sorted (the Farey sequence F_n)."""
    s = {Fraction(a, b) for b in range(1, n + 1) for a in range(0, b + 1)}
    return sorted(s)


_CACHE = {}


def enumerate_emitted(Pp, Qp, T, denom, draft_law=None, runner=None):
    """Exact distribution of the first K+1 emitted tokens for prefix-independent rows.

    Pp: K+1 rows of rational probabilities, Qp: K rows (the q the verifier is given).
    Every draft tuple is weighted by prod draft_law_i(x_i) (default: q itself); every
    uniform coordinate is swept over the intervals between consecutive members of the
    Farey sequence F_denom. All probabilities have denominators dividing ``denom``, so
    every ratio p/q and every normalised CDF point of any residual lies in F_denom: the
    oracle's output is constant on each interval and its midpoint decides it. Tokens the
    cycle does not emit are continued with p_{n+2}..p_{K+1}, as a prefix-independent
    target would produce them.

    ``runner(zP, zQ, drafts, T, u)`` runs the verify step on the batch of every (draft tuple,
    uniform cell) pair (float64 logits, [n, K] drafts, [n, K+1] float32-representable
    uniforms) and returns an object with ``n_accepted`` and ``tokens``; default: the oracle.
    Returns (law, result): the emitted law as {token tuple: Fraction} and the runner's
    result, whose rows are ordered draft tuple first, then uniform cell.
    """
    law = Qp if draft_law is None else draft_law
    K = len(Qp)
    V = len(Pp[0])
    zP = np.stack([logits_of(r, T) for r in Pp])[None]
    zQ = np.stack([logits_of(r, T) for r in Qp])[None]
    F = farey(denom)
    cells = [((F[k] + F[k + 1]) / 2, F[k + 1] - F[k]) for k in range(len(F) - 1)]
    ucells = list(itertools.product(cells, repeat=K + 1))
    # midpoints rounded to float32 (the GPU's uniform type); they stay >= 1/(2 denom^2) - 2^-25
    # from every Farey point, so the rounding changes no decision
    u_one = np.asarray([[float(c[0]) for c in us] for us in ucells], dtype=np.float32)
    u_one = u_one.astype(np.float64)
    w_one = []
    for us in ucells:
        w = Fraction(1)
        for c in us:
            w *= c[1]
        w_one.append(w)
    drafts_all = [x for x in itertools.product(range(V), repeat=K)
                  if all(Qp[i][x[i]] > 0 or law[i][x[i]] > 0 for i in range(K))]
    nu = len(ucells)
    run = runner or _oracle_runner
    key = (repr(Pp), repr(Qp), T, denom, tuple(drafts_all), run)
    if key not in _CACHE:
        n = nu * len(drafts_all)
        d = np.repeat(np.asarray(drafts_all, dtype=np.int64), nu, axis=0)
        u = np.tile(u_one, (len(drafts_all), 1))
        _CACHE[key] = run(np.repeat(zP, n, axis=0), np.repeat(zQ, n, axis=0), d, T, u)
    res = _CACHE[key]
    emitted_w = {}
    for a, x in enumerate(drafts_all):
        wx = Fraction(1)
        for i in range(K):
            wx *= law[i][x[i]]
        if not wx:
            continue
        acc = {}
        for k in range(nu):
            row = a * nu + k
            nb = int(res.n_accepted[row])
            key = tuple(int(t) for t in res.tokens[row, : nb + 1])
            acc[key] = acc.get(key, Fraction(0)) + w_one[k]
        for key, w in acc.items():
            emitted_w[key] = emitted_w.get(key, Fraction(0)) + wx * w
    dist = {}
    for emitted, w in emitted_w.items():
        nb = len(emitted) - 1
        for tail in itertools.product(range(V), repeat=K - nb):
            ww = w
            for m, t in enumerate(tail):
                ww *= Pp[nb + 1 + m][t]
            if ww:
                dist[emitted + tail] = dist.get(emitted + tail, Fraction(0)) + ww
    return dist, res


def _oracle_runner(zP, zQ, d, T, u):
    return ora.speculative_sample_accept(zP, zQ, d, T, u)


def product_dist(Pp):
    out = {}
    for s in itertools.product(range(len(Pp[0])), repeat=len(Pp)):
        w = Fraction(1)
        for r, t in enumerate(s):
            w *= Pp[r][t]
        if w:
            out[s] = w
    return out
