"""Pins of the oracle's early-exit step (``early_exit_accept``): rows are read in draft order
and each sequence stops at its first rejection.

Checked against the full step (itself pinned by exact enumeration, a greedy decode loop and
library inverse-CDF draws): on blocks whose rows are all usable the two agree on every
output; rows after the first rejection can be poisoned without effect (while the full step
reports them); a bad row at or before the stop, or a bad bonus row after a full accept, is
an error; a bad draft id reads nothing.
"""

import numpy as np
import pytest

from oracle import accept_ref as ora


def _block(seed, B, K, V, noise=1.0):
    rng = np.random.default_rng(seed)
    P = rng.normal(0, 2, size=(B, K + 1, V))
    Q = P[:, :K] + rng.normal(0, noise, size=(B, K, V))
    u = rng.random((B, K + 1))
    am = P.argmax(axis=2)
    drafts = rng.integers(0, V, size=(B, K))
    for b in range(B):  # long accepted prefixes are common, as in real blocks
        m = rng.integers(0, K + 1)
        drafts[b, :m] = am[b, :m]
    return P, Q, drafts, u


def _full(P, Q, d, T, u):
    return ora.speculative_sample_accept(P, Q, d, T, u)


@pytest.mark.parametrize("K", [0, 1, 3, 7])
@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
def test_usable_blocks_equal_the_full_step(K, T):
    P, Q, d, u = _block(11 + K, 40, K, 50)
    a = ora.early_exit_accept(P, Q, d, T, u)
    f = _full(P, Q, d, T, u)
    assert np.array_equal(a.n_accepted, f.n_accepted)
    assert np.array_equal(a.tokens, f.tokens)
    assert np.array_equal(a.next_token, f.next_token)
    assert np.array_equal(a.status, f.status)
    if T > 0:
        np.testing.assert_array_equal(a.resid_mass, f.resid_mass)
        for b in range(P.shape[0]):
            j = int(f.n_accepted[b])
            t = min(j + 1, K)
            assert np.array_equal(a.p_draft[b, :t], f.p_draft[b, :t])
            assert np.array_equal(a.q_draft[b, :t], f.q_draft[b, :t])
            assert np.all(np.isnan(a.p_draft[b, t:])) and np.all(np.isnan(a.q_draft[b, t:]))


@pytest.mark.parametrize("T", [0.0, 1.0])
@pytest.mark.parametrize("poison", [np.nan, np.inf, -np.inf])
def test_rows_after_the_first_rejection_are_not_read(T, poison):
    K = 6
    P, Q, d, u = _block(21, 60, K, 40)
    f = _full(P, Q, d, T, u)
    P2, Q2 = P.copy(), Q.copy()
    cut = 0
    for b in range(P.shape[0]):
        j = int(f.n_accepted[b])
        if j < K:
            P2[b, j + 1:] = poison  # rows j+1..K, the bonus row among them
            Q2[b, j + 1:] = poison
            cut += 1
    assert cut > 20
    a = ora.early_exit_accept(P2, Q2, d, T, u)
    assert np.array_equal(a.tokens, f.tokens) and np.array_equal(a.n_accepted, f.n_accepted)
    assert np.all(a.status == f.status)
    g = _full(P2, Q2, d, T, u)  # the full step reads them and reports them
    assert np.sum(g.status == ora.STATUS_NONFINITE) == cut


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_bad_rows_up_to_the_stop_are_errors(T):
    K = 5
    P, Q, d, u = _block(31, 60, K, 40)
    f = _full(P, Q, d, T, u)
    rng = np.random.default_rng(3)
    P2, Q2 = P.copy(), Q.copy()
    want = np.zeros(P.shape[0], dtype=bool)
    for b in range(P.shape[0]):
        j = int(f.n_accepted[b])
        if b % 3 == 0:
            continue
        i = int(rng.integers(0, j + 1))          # a row at or before the stop
        if i == K or (b % 3 == 1 or T == 0):
            P2[b, i, rng.integers(0, 40)] = np.nan
        else:
            Q2[b, i, :] = -np.inf               # no finite value
        want[b] = True
    a = ora.early_exit_accept(P2, Q2, d, T, u)
    assert np.array_equal(a.status == ora.STATUS_NONFINITE, want)
    assert np.all(a.n_accepted[want] == 0) and np.all(a.tokens[want] == -1)
    assert np.all(a.next_token[want] == -1)
    assert np.array_equal(a.tokens[~want], f.tokens[~want])


def test_bad_draft_id_reads_nothing():
    K = 3
    P, Q, d, u = _block(41, 4, K, 20)
    d[1, 2] = 20
    d[2, 0] = -1
    P[1:3] = np.nan
    for T in (0.0, 1.0):
        a = ora.early_exit_accept(P, Q, d, T, u)
        assert list(a.status) == [0, ora.STATUS_BAD_DRAFT, ora.STATUS_BAD_DRAFT, 0]


def test_exact_enumeration_is_lossless():
    """V = 4, K = 2, probabilities in eighths: over every draft pair x ~ q_1 x q_2 and every
    cell of the three uniforms between consecutive members of the Farey sequence F_8 (all
    decision and CDF boundaries lie there), the tokens early_exit_accept emits, continued
    with p_{n+2}.. where it stops early, follow p_1 x p_2 x p_3 exactly."""
    import itertools
    from fractions import Fraction

    F8 = lambda *xs: [Fraction(x, 8) for x in xs]  # noqa: E731
    # both residuals keep two tokens (max(p_1 - q_1, 0) = (2, 0, 1, 0)/8, max(p_2 - q_2, 0) =
    # (0, 2, 1, 0)/8), so the draw's uniform decides the token and a draw with the wrong
    # uniform changes the law
    Pp = [F8(3, 2, 2, 1), F8(1, 3, 2, 2), F8(1, 2, 3, 2)]
    Qp = [F8(1, 3, 1, 3), F8(2, 1, 1, 4)]
    V, K = 4, 2
    with np.errstate(divide="ignore"):
        zP = np.log(np.array([[float(x) for x in r] for r in Pp]))
        zQ = np.log(np.array([[float(x) for x in r] for r in Qp]))
    F = sorted({Fraction(a, b) for b in range(1, 9) for a in range(b + 1)})
    cells = [((F[k] + F[k + 1]) / 2, F[k + 1] - F[k]) for k in range(len(F) - 1)]
    runs = [(x, us) for x in itertools.product(range(V), repeat=K)
            if Qp[0][x[0]] * Qp[1][x[1]] > 0
            for us in itertools.product(cells, repeat=K + 1)]
    n = len(runs)
    d = np.array([x for x, _ in runs])
    u = np.array([[float(c[0]) for c in us] for _, us in runs])
    res = ora.early_exit_accept(np.repeat(zP[None], n, 0), np.repeat(zQ[None], n, 0), d, 1.0, u)
    assert np.all(res.status == 0)
    law = {}
    for r, (x, us) in enumerate(runs):
        w = Qp[0][x[0]] * Qp[1][x[1]]
        for c in us:
            w *= c[1]
        nb = int(res.n_accepted[r])
        emitted = tuple(int(t) for t in res.tokens[r, : nb + 1])
        for tail in itertools.product(range(V), repeat=K - nb):
            ww = w
            for m, t in enumerate(tail):
                ww *= Pp[nb + 1 + m][t]
            if ww:
                law[emitted + tail] = law.get(emitted + tail, Fraction(0)) + ww
    want = {}
    for s in itertools.product(range(V), repeat=K + 1):
        w = Pp[0][s[0]] * Pp[1][s[1]] * Pp[2][s[2]]
        if w:
            want[s] = w
    assert law == want
