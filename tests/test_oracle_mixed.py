"""Pins of the oracle's mixed serving batch (per-sequence draft counts and temperatures).

Sequence b of a mixed batch verifies its first K_b drafts at its own temperature T_b
(T_b == 0: greedy); rows, drafts and uniforms past K_b are never read. Each test checks
``mixed_accept`` against something other than itself: an exact rational enumeration of
the emitted law, a plain argmax decode loop, or the library inverse CDF
(``np.searchsorted`` on ``np.cumsum``).
"""

import itertools
from fractions import Fraction

import numpy as np

from oracle import accept_ref as ora

F8 = lambda *xs: [Fraction(x, 8) for x in xs]  # noqa: E731


def _logits_of(probs):
    p = np.asarray([float(x) for x in probs])
    with np.errstate(divide="ignore"):
        return np.log(p)


def _farey(n):
    return sorted({Fraction(a, b) for b in range(1, n + 1) for a in range(0, b + 1)})


def test_truncated_block_is_lossless_and_ignores_what_lies_past_it():
    """K_b = 1 inside a K = 2 block. The unused P row and Q row are NaN, the unused draft
    is out of range and the unused uniform is a fixed junk value: the two emitted tokens
    must still follow p_1 x p_2 exactly, over every draft x_0 ~ q_1 and every cell of the
    two uniforms that matter (u_0 for the test, u_1 = u[b, K_b] for the draw)."""
    Pp = [F8(4, 2, 1, 1), F8(1, 1, 2, 4)]
    Qp = [F8(2, 3, 2, 1)]
    V, K = 4, 2
    zP = np.full((K + 1, V), np.nan)
    zP[0], zP[1] = _logits_of(Pp[0]), _logits_of(Pp[1])
    zQ = np.full((K, V), np.nan)
    zQ[0] = _logits_of(Qp[0])
    F = _farey(8)
    cells = [((F[k] + F[k + 1]) / 2, F[k + 1] - F[k]) for k in range(len(F) - 1)]
    rows = []
    for x in range(V):
        for c0, c1 in itertools.product(cells, repeat=2):
            rows.append((x, c0, c1))
    n = len(rows)
    d = np.array([[x, -5] for x, _, _ in rows])
    u = np.array([[float(c0[0]), float(c1[0]), 0.123] for _, c0, c1 in rows])
    res = ora.mixed_accept(np.repeat(zP[None], n, 0), np.repeat(zQ[None], n, 0), d,
                           np.full(n, 1), np.full(n, 1.0), u)
    assert np.all(res.status == 0)
    law = {}
    for r, (x, c0, c1) in enumerate(rows):
        w = Qp[0][x] * c0[1] * c1[1]
        if not w:
            continue
        nb = int(res.n_accepted[r])
        assert nb in (0, 1) and np.all(res.tokens[r, nb + 1:] == -1)
        emitted = tuple(int(t) for t in res.tokens[r, : nb + 1])
        tails = itertools.product(range(V), repeat=1 - nb)
        for tail in tails:
            ww = w
            for m, t in enumerate(tail):
                ww *= Pp[nb + 1 + m][t]
            if ww:
                law[emitted + tail] = law.get(emitted + tail, Fraction(0)) + ww
    want = {(a, b): Pp[0][a] * Pp[1][b] for a in range(V) for b in range(V)
            if Pp[0][a] * Pp[1][b]}
    assert law == want


def test_greedy_sequences_follow_an_argmax_decode_loop():
    rng = np.random.default_rng(5)
    B, K, V = 40, 6, 50
    P = rng.normal(0, 2, size=(B, K + 1, V))
    drafts = rng.integers(0, V, size=(B, K))
    kb = rng.integers(0, K + 1, size=B)
    am = P.argmax(axis=2)
    for b in range(B):  # make long accepted prefixes common
        m = rng.integers(0, K + 1)
        drafts[b, :m] = am[b, :m]
        P[b, kb[b] + 1:] = np.nan       # never read
        drafts[b, kb[b]:] = V + 7       # never read
    res = ora.mixed_accept(P, None, drafts, kb, np.zeros(B), None)
    for b in range(B):
        j = 0
        while j < kb[b] and drafts[b, j] == np.nanargmax(P[b, j]):
            j += 1
        assert res.status[b] == 0 and res.n_accepted[b] == j
        assert list(res.tokens[b, :j]) == list(drafts[b, :j])
        assert res.tokens[b, j] == np.nanargmax(P[b, j]) == res.next_token[b]
        assert np.all(res.tokens[b, j + 1:] == -1)


def test_zero_drafts_draws_p1_with_its_own_uniform():
    """K_b = 0: no test is taken and the token is the library inverse CDF of p_1 at
    u[b, 0], whatever the rest of the block holds."""
    rng = np.random.default_rng(6)
    B, K, V = 30, 4, 40
    P = rng.normal(0, 2, size=(B, K + 1, V))
    Q = rng.normal(0, 2, size=(B, K, V))
    u = rng.random((B, K + 1))
    T = rng.choice([0.5, 1.0, 1.7], size=B)
    P[:, 1:] = np.inf  # never read
    res = ora.mixed_accept(P, Q, np.zeros((B, K), dtype=int), np.zeros(B, dtype=int), T, u)
    for b in range(B):
        z = P[b, 0] / T[b]
        p = np.exp(z - z.max())
        c = np.cumsum(p)
        v = int(np.searchsorted(c, u[b, 0] * c[-1], side="right"))
        assert res.status[b] == 0 and res.n_accepted[b] == 0 and res.tokens[b, 0] == v
        assert np.all(res.tokens[b, 1:] == -1)


def test_bonus_row_is_row_kb():
    """q == p on the used rows: every one of the K_b drafts is accepted and the bonus is the
    library inverse CDF of p_{K_b+1} (row K_b) at u[b, K_b]."""
    rng = np.random.default_rng(7)
    B, K, V = 20, 5, 30
    P = rng.normal(0, 2, size=(B, K + 1, V))
    Q = P[:, :K].copy()
    kb = rng.integers(1, K + 1, size=B)
    u = rng.random((B, K + 1))
    drafts = rng.integers(0, V, size=(B, K))
    res = ora.mixed_accept(P, Q, drafts, kb, np.ones(B), u)
    for b in range(B):
        k = int(kb[b])
        c = np.cumsum(np.exp(P[b, k] - P[b, k].max()))
        v = int(np.searchsorted(c, u[b, k] * c[-1], side="right"))
        assert res.n_accepted[b] == k and res.tokens[b, k] == v == res.next_token[b]
        assert list(res.tokens[b, :k]) == list(drafts[b, :k])
        assert res.resid_mass[b] == 1.0


def test_bad_parameters_are_errors_of_their_sequence_only():
    rng = np.random.default_rng(8)
    B, K, V = 7, 3, 20
    P = rng.normal(0, 2, size=(B, K + 1, V))
    Q = rng.normal(0, 2, size=(B, K, V))
    u = rng.random((B, K + 1))
    drafts = rng.integers(0, V, size=(B, K))
    kb = np.array([-1, K + 1, 2, 2, 2, 2, 1])
    T = np.array([1.0, 1.0, -0.5, np.nan, np.inf, 0.0, 0.9])
    res = ora.mixed_accept(P, Q, drafts, kb, T, u)
    for b in range(5):
        assert res.status[b] == ora.STATUS_BAD_PARAM
        assert res.n_accepted[b] == 0 and res.next_token[b] == -1
        assert np.all(res.tokens[b] == -1)
    assert res.status[5] == 0 and res.status[6] == 0
    g = ora.greedy_accept(P[5:6, :3], drafts[5:6, :2])
    assert res.n_accepted[5] == g.n_accepted[0] and res.tokens[5, 0] == g.tokens[0, 0]


def test_uniform_batch_equals_the_single_policy_calls():
    """Every K_b = K and one temperature: the single-policy step (the same arithmetic, so
    this only checks the layout of the mixed results)."""
    rng = np.random.default_rng(9)
    B, K, V = 6, 3, 25
    P = rng.normal(0, 2, size=(B, K + 1, V))
    Q = rng.normal(0, 2, size=(B, K, V))
    u = rng.random((B, K + 1))
    drafts = rng.integers(0, V, size=(B, K))
    for T in (0.0, 0.8):
        a = ora.mixed_accept(P, Q, drafts, None, np.full(B, T), u)
        b = ora.speculative_sample_accept(P, Q, drafts, T, u)
        assert np.array_equal(a.tokens, b.tokens) and np.array_equal(a.n_accepted, b.n_accepted)
