"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test fixes the oracle to something the pages or the mathematics determine:
exact losslessness (the emitted tokens are distributed exactly as the target's,
dspark-mlx wheel adapter.py docstring and the DeepSeek-V4-Flash DSpark drafter card),
identity with plain sequential greedy decoding (mlx-dspark README, "How it works", and
its benchmark.py greedy loop), library inverse-CDF draws, the closed-form acceptance
rate of speculative sampling, a chi-square goodness of fit, and hand-worked examples.
"""

import os
from fractions import Fraction

import numpy as np
import pytest
from scipy import special, stats

from oracle import accept_ref as ora

import enumeration as en
from lossless_draft_verification_speculative_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

F8 = lambda *xs: [Fraction(x, 8) for x in xs]  # noqa: E731


# --------------------------------------------------------- losslessness

def test_enumeration_lossless_exact():
    """V=4, K=2: the joint law of the K+1 emitted tokens equals p_1 x p_2 x p_3 exactly."""
    Pp = [F8(4, 2, 1, 1), F8(1, 1, 2, 4), F8(2, 2, 3, 1)]
    Qp = [F8(2, 3, 2, 1), F8(4, 2, 1, 1)]
    got, _ = en.enumerate_emitted(Pp, Qp, 1.0, 8)
    assert got == en.product_dist(Pp)


@pytest.mark.parametrize("T", [0.5, 2.0])
def test_enumeration_lossless_exact_tempered(T):
    """Same check at T != 1 (logits log(p) * T), on quarter-denominator rows."""
    F4 = lambda *xs: [Fraction(x, 4) for x in xs]  # noqa: E731
    Pp = [F4(2, 1, 1, 0), F4(0, 1, 1, 2), F4(1, 1, 1, 1)]
    Qp = [F4(1, 1, 1, 1), F4(2, 2, 0, 0)]
    got, _ = en.enumerate_emitted(Pp, Qp, T, 4)
    assert got == en.product_dist(Pp)


def test_enumeration_lossless_with_masked_tokens():
    """Zero-probability tokens (logit -inf) in p and in q: still exactly lossless."""
    Pp = [F8(0, 4, 4, 0), F8(1, 0, 3, 4), F8(0, 0, 0, 8)]
    Qp = [F8(2, 2, 2, 2), F8(0, 4, 0, 4)]
    got, _ = en.enumerate_emitted(Pp, Qp, 1.0, 8)
    assert got == en.product_dist(Pp)


def test_enumeration_detects_a_wrong_rule():
    """The enumeration has power: a draft law that is not q breaks the product form.

    Weighting the same oracle runs by a different draft law (uniform instead of q) must
    not give p_1 x p_2 x p_3. This guards the pin itself against being vacuous.
    """
    Pp = [F8(4, 2, 1, 1), F8(1, 1, 2, 4), F8(2, 2, 3, 1)]
    Qp_true = [F8(2, 3, 2, 1), F8(4, 2, 1, 1)]
    Qp_fake = [F8(2, 2, 2, 2), F8(2, 2, 2, 2)]
    got, _ = en.enumerate_emitted(Pp, Qp_true, 1.0, 8)
    bad, _ = en.enumerate_emitted(Pp, Qp_true, 1.0, 8, draft_law=Qp_fake)
    assert got == en.product_dist(Pp)
    assert bad != en.product_dist(Pp)


# ---------------------------------------------------------- greedy

class _FakeTarget:
    """A prefix-dependent next-token distribution: logits looked up by the whole prefix."""

    def __init__(self, V, seed, ties=False):
        self.V, self.seed, self.ties = V, seed, ties
        self.cache = {}

    def logits(self, prefix):
        key = tuple(prefix)
        if key not in self.cache:
            rng = np.random.default_rng([self.seed, len(key)] + list(key))
            z = np.round(rng.normal(0, 1, self.V), 1 if self.ties else 12)
            self.cache[key] = z
        return self.cache[key]


@pytest.mark.parametrize("ties", [False, True])
def test_greedy_equals_sequential_greedy_decoding(ties):
    """Committed tokens equal plain greedy decoding (one target forward per token)."""
    V, K = 16, 5
    rng = np.random.default_rng(7)
    for trial in range(200):
        tgt = _FakeTarget(V, trial, ties)
        ctx = list(rng.integers(0, V, 3))
        # plain greedy decoding, K+1 tokens, first-occurrence argmax (numpy)
        seq = []
        for _ in range(K + 1):
            seq.append(int(np.argmax(tgt.logits(ctx + seq))))
        # drafts: the greedy sequence with a random corruption point (or none)
        m = int(rng.integers(0, K + 1))
        d = list(seq[:K])
        if m < K:
            d[m] = (d[m] + 1 + int(rng.integers(0, V - 1))) % V
        # verify block: row r scores position r given the drafts before it
        P = np.stack([tgt.logits(ctx + d[:r]) for r in range(K + 1)])[None]
        res = ora.greedy_accept(P, np.asarray([d]))
        n = int(res.n_accepted[0])
        assert n == m
        assert list(res.tokens[0, : n + 1]) == seq[: n + 1]
        assert all(t == -1 for t in res.tokens[0, n + 1:])
        assert int(res.next_token[0]) == seq[n]


def test_greedy_ties_lowest_index_and_signed_zero():
    ninf = -np.inf
    rows = [
        [0.5, 2.0, 2.0, -1.0, 2.0],
        [ninf, ninf, 0.0, ninf, -0.0],
        [ninf, ninf, -0.0, ninf, 0.0],
        [3.0, 3.0, 3.0, 3.0, 3.0],
    ]
    for r in rows:
        z = np.asarray(r)
        assert ora.row_argmax(z) == int(np.argmax(z))
    assert ora.row_argmax(np.asarray(rows[1])) == 2
    assert ora.row_argmax(np.asarray(rows[2])) == 2


def test_sampling_at_T0_is_greedy():
    w = wl.WORKLOADS["tiny"]
    P, Q = wl.logits(w)
    d = wl.drafts(w, Q, 0.0)
    u = wl.uniforms(w)
    Pf, Qf = wl.as_float64(P, w.dtype), wl.as_float64(Q, w.dtype)
    a = ora.speculative_sample_accept(Pf, Qf, d, 0.0, u)
    g = ora.greedy_accept(Pf, d)
    assert np.array_equal(a.tokens, g.tokens) and np.array_equal(a.n_accepted, g.n_accepted)
    assert int(g.n_accepted[0]) == w.K or g.tokens[0, g.n_accepted[0]] != d[0, g.n_accepted[0]]


# ------------------------------------------------- invariants, closed forms

def test_q_equal_p_accepts_everything():
    rng = np.random.default_rng(3)
    B, K, V = 64, 6, 50
    P = rng.normal(0, 2, (B, K + 1, V))
    Q = P[:, :K].copy()
    for T in (0.6, 1.0, 1.7):
        d = rng.integers(0, V, (B, K))
        u = rng.random((B, K + 1))
        res = ora.speculative_sample_accept(P, Q, d, T, u)
        assert np.all(res.n_accepted == K)
        assert np.array_equal(res.tokens[:, :K], d)


def test_bonus_is_library_inverse_cdf():
    """All drafts accepted (q == p): the bonus is searchsorted(cumsum(p_K), u * sum)."""
    rng = np.random.default_rng(4)
    B, K, V = 200, 3, 37
    P = rng.normal(0, 2, (B, K + 1, V))
    T = 0.8
    d = rng.integers(0, V, (B, K))
    u = rng.random((B, K + 1))
    res = ora.speculative_sample_accept(P, P[:, :K].copy(), d, T, u)
    for b in range(B):
        p = special.softmax(P[b, K] / T)
        c = np.cumsum(p)
        assert res.next_token[b] == np.searchsorted(c, u[b, K] * c[-1], side="right")


def test_point_mass_draft_rejects_to_p_without_x():
    """q_0 is a point mass on x: accept iff u_0 < p(x); on rejection the residual is p with
    x removed, so the correction is a library inverse-CDF draw from that."""
    rng = np.random.default_rng(5)
    V, K = 23, 1
    for trial in range(300):
        zP = rng.normal(0, 1.5, (1, K + 1, V))
        x = int(rng.integers(0, V))
        zQ = np.full((1, K, V), -np.inf)
        zQ[0, 0, x] = 0.0
        u = rng.random((1, K + 1))
        res = ora.speculative_sample_accept(zP, zQ, np.asarray([[x]]), 1.0, u)
        p0 = special.softmax(zP[0, 0])
        if u[0, 0] < p0[x]:
            assert res.n_accepted[0] == 1
            c = np.cumsum(special.softmax(zP[0, 1]))
            assert res.next_token[0] == np.searchsorted(c, u[0, 1] * c[-1], side="right")
        else:
            assert res.n_accepted[0] == 0
            w = p0.copy()
            w[x] = 0.0
            c = np.cumsum(w)
            assert res.next_token[0] == np.searchsorted(c, u[0, 1] * c[-1], side="right")
            assert res.next_token[0] != x


def test_temperature_scaling_identity():
    """softmax(z / T) only depends on z / T: (z, T) and (2z, 2T) give identical results."""
    rng = np.random.default_rng(6)
    B, K, V = 40, 4, 30
    P = rng.normal(0, 2, (B, K + 1, V))
    Q = P[:, :K] + rng.normal(0, 1, (B, K, V))
    d = rng.integers(0, V, (B, K))
    u = rng.random((B, K + 1))
    a = ora.speculative_sample_accept(P, Q, d, 0.7, u)
    b = ora.speculative_sample_accept(2 * P, 2 * Q, d, 1.4, u)
    assert np.array_equal(a.tokens, b.tokens)
    np.testing.assert_allclose(a.p_draft, b.p_draft, rtol=1e-13)


def test_softmax_matches_chosen_probabilities():
    probs = [Fraction(1, 2), Fraction(1, 4), Fraction(1, 8), Fraction(1, 8), Fraction(0)]
    for T in (0.5, 1.0, 3.0):
        p = ora.softmax(en.logits_of(probs, T), T)
        np.testing.assert_allclose(p, [float(x) for x in probs], rtol=1e-15, atol=0)


def test_acceptance_rate_closed_form():
    """E[n] = sum_{k=1..K} prod_{i<k} alpha_i with alpha_i = sum_v min(p_i, q_i)."""
    rng = np.random.default_rng(8)
    K, V, N, T = 4, 40, 4000, 1.0
    zP = rng.normal(0, 2, (1, K + 1, V))
    zQ = zP[:, :K] + rng.normal(0, 1.0, (1, K, V))
    p = [special.softmax(zP[0, i] / T) for i in range(K + 1)]
    q = [special.softmax(zQ[0, i] / T) for i in range(K)]
    alpha = [np.minimum(p[i], q[i]).sum() for i in range(K)]
    expect = sum(np.prod(alpha[:k]) for k in range(1, K + 1))
    # drafts ~ q_i by inverse CDF with an independent generator (library searchsorted)
    d = np.stack([[np.searchsorted(np.cumsum(q[i]), rng.random(), side="right")
                   for i in range(K)] for _ in range(N)])
    u = rng.random((N, K + 1))
    res = ora.speculative_sample_accept(np.repeat(zP, N, 0), np.repeat(zQ, N, 0), d, T, u)
    n = res.n_accepted.astype(np.float64)
    assert abs(n.mean() - expect) < 4 * n.std(ddof=1) / np.sqrt(N)


def test_chi_square_first_token_tiny_workload():
    """Tiny workload (B1 K3 V64 fp32, 1000 cycles, T=1): first emitted token ~ p_1."""
    w = wl.WORKLOADS["tiny"]
    P, Q, d, u = wl.tiny_cycles(w, 1000)
    res = ora.speculative_sample_accept(wl.as_float64(P, w.dtype), wl.as_float64(Q, w.dtype),
                                        d, 1.0, u)
    first = res.tokens[:, 0]
    p1 = special.softmax(wl.as_float64(P[0, 0], w.dtype))
    obs = np.bincount(first, minlength=w.V).astype(np.float64)
    exp = p1 * len(first)
    order = np.argsort(exp)
    # pool the smallest bins until every pooled bin expects at least 5
    bins_o, bins_e, acc_o, acc_e = [], [], 0.0, 0.0
    for v in order:
        acc_o += obs[v]
        acc_e += exp[v]
        if acc_e >= 5:
            bins_o.append(acc_o)
            bins_e.append(acc_e)
            acc_o = acc_e = 0.0
    if acc_e > 0:
        bins_o[-1] += acc_o
        bins_e[-1] += acc_e
    pval = stats.chisquare(bins_o, bins_e).pvalue
    assert pval > 1e-3


# --------------------------------------------------------- error semantics

def test_bad_draft_and_nonfinite_rows():
    rng = np.random.default_rng(9)
    B, K, V = 5, 3, 12
    P = rng.normal(0, 1, (B, K + 1, V))
    Q = rng.normal(0, 1, (B, K, V))
    d = rng.integers(0, V, (B, K))
    u = rng.random((B, K + 1))
    d[0, 2] = V           # out of range (even past a rejection point)
    P[1, 3, 4] = np.nan   # NaN in the bonus row
    Q[2, 1, :] = -np.inf  # a draft row with no finite value
    P[3, 0, :5] = -np.inf  # masked tokens are allowed
    P[4, 2, 7] = np.inf
    for res in (ora.speculative_sample_accept(P, Q, d, 1.0, u), ora.greedy_accept(P, d)):
        for b in (0, 1, 4):
            assert res.status[b] != 0 and res.n_accepted[b] == 0 and res.next_token[b] == -1
            assert np.all(res.tokens[b] == -1)
        assert res.status[3] == 0 and res.next_token[3] >= 0
    assert ora.speculative_sample_accept(P, Q, d, 1.0, u).status[2] & ora.STATUS_NONFINITE
    assert ora.greedy_accept(P, d).status[2] == 0  # greedy never reads Q


# ------------------------------------------------------------- golden

def _load_golden(name):
    cases = []
    cur = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line == "---":
                if cur:
                    cases.append(cur)
                cur = {}
                continue
            k, v = line.split("=", 1)
            cur[k.strip()] = v.strip()
    if cur:
        cases.append(cur)
    return cases


def _fr_row(s):
    return [Fraction(t) for t in s.split()]


def test_golden_hand_worked_examples():
    cases = _load_golden("hand_worked_v4_k2.txt")
    assert len(cases) >= 4
    for c in cases:
        K = int(c["K"])
        Pp = [_fr_row(c[f"p{r + 1}"]) for r in range(K + 1)]
        T = float(c.get("T", "1"))
        zP = np.stack([en.logits_of(r, T) for r in Pp])[None]
        d = np.asarray([[int(t) for t in c["drafts"].split()]])
        u = np.asarray([[float(t) for t in c["u"].split()]])
        if c["policy"] == "greedy":
            res = ora.greedy_accept(zP, d)
        else:
            Qp = [_fr_row(c[f"q{i + 1}"]) for i in range(K)]
            zQ = np.stack([en.logits_of(r, T) for r in Qp])[None]
            res = ora.speculative_sample_accept(zP, zQ, d, T, u)
        assert int(res.n_accepted[0]) == int(c["n_accepted"]), c
        assert [int(t) for t in res.tokens[0]] == [int(t) for t in c["tokens"].split()], c
        if "resid_mass" in c:
            assert abs(res.resid_mass[0] - float(Fraction(c["resid_mass"]))) < 1e-12


def test_near_boundary_flag():
    """A uniform placed 1e-9 from the accept boundary is flagged; 1e-3 away is not."""
    Pp = [F8(4, 2, 1, 1), F8(2, 2, 2, 2)]
    Qp = [F8(2, 2, 2, 2)]
    zP = np.stack([en.logits_of(r) for r in Pp])[None]
    zQ = np.stack([en.logits_of(r) for r in Qp])[None]
    d = np.asarray([[2]])  # ratio (1/8)/(2/8) = 0.5
    near = ora.speculative_sample_accept(zP, zQ, d, 1.0, np.asarray([[0.5 - 1e-9, 0.3]]))
    far = ora.speculative_sample_accept(zP, zQ, d, 1.0, np.asarray([[0.499, 0.3]]))
    assert near.near_boundary()[0] and not far.near_boundary()[0]


def test_draw_law_and_cdf_interval():
    """draw_law after a rejection under a point-mass q is p without x (library softmax), and
    cdf_interval brackets exactly the uniforms whose library inverse-CDF draw is v."""
    rng = np.random.default_rng(11)
    V, K = 17, 2
    zP = rng.normal(0, 1.5, (K + 1, V))
    zQ = np.full((K, V), -np.inf)
    zQ[0, 5] = 0.0
    zQ[1] = rng.normal(0, 1.5, V)
    w = ora.draw_law(zP, zQ, 0, 1.0)
    p0 = special.softmax(zP[0])
    want = p0.copy()
    want[5] = 0.0
    np.testing.assert_allclose(w, want, rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(ora.draw_law(zP, zQ, K, 1.0), special.softmax(zP[K]), rtol=1e-13)
    c = np.cumsum(want)
    for uu in rng.random(200):
        v = int(np.searchsorted(c, uu * c[-1], side="right"))
        lo, hi = ora.cdf_interval(want, v)
        assert lo <= uu < hi
