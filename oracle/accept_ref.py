"""CPU float64 oracle of the DSpark block verify/accept step.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may import or run this module. The product path never
does: it shares no code with this file and imports nothing from ``oracle/``.

What it computes, and where that comes from:

* The logit block. Row 0 of P is p_1, the base distribution for the first drafted
  token, produced by the anchor step; rows 1..K are p_2..p_{K+1} from one verify
  forward over the K drafts; row K is the bonus position. Page "dspark-mlx
  0.1.0__py3-none-any.whl", ``dspark_mlx/adapter.py`` module docstring ("Logit
  conventions") and the ``StepOut`` / ``BlockOut`` dataclasses.
* The two accept policies, ``greedy_accept`` and ``speculative_sample_accept``, and the
  ``AcceptResult`` they return, are named by the same wheel's ``dspark_mlx/__init__.py``
  (imports from ``.verify``); their bodies are not on the pages. The wheel calls the
  policy lossless (adapter.py docstring), the mlx-dspark README ("How it works") calls
  greedy verification identical to plain greedy decoding up to near-tie breaking, and
  the DeepSeek-V4-Flash DSpark drafter model card calls decoding lossless because the
  target's verify forward is the only token source.
* The rule itself is the published speculative-sampling rule (Leviathan, Kalman &
  Matias 2023; Chen et al. 2023): accept draft x_i with probability min(1, p_i(x_i) /
  q_i(x_i)); at the first rejection draw from normalize(max(p_i - q_i, 0)); when every
  draft is accepted draw the bonus token from p_{K+1}. Greedy: accept while the draft
  equals the base argmax, then emit the argmax of the first mismatching (or bonus) row.

Readings where the pages are silent:
  temperature divides both P and Q logits; T == 0 means greedy; u[b, i] tests draft i
  and u[b, K] is the single draw for the resample or bonus token; accept iff
  u * q(x) < p(x) (strict; q == 0 < p accepts); the inverse CDF runs in ascending token
  id and returns the smallest v with C(v) > u * Z; argmax ties go to the lowest index
  and -0.0 equals +0.0; a zero residual mass after a rejection (possible only through
  rounding) falls back to p_j; a draft id outside [0, V) or a row holding NaN or +inf,
  or no finite value at all, makes the whole sequence an error (n = 0, tokens -1).

Mixed serving batches (``mixed_accept``). The mlx-dspark README ("Tuning") truncates the
block per step through the drafter's confidence head (``--confidence-threshold``) or caps
it (``--max-draft``), and the ds4 fork the DeepSeek-V4-Flash drafter card names serves
batches. So each sequence b of a batch may carry its own draft count K_b <= K and its
own temperature T_b (T_b == 0: greedy). Reading: sequence b is the single-policy step on
its own truncated block, P rows 0..K_b (row K_b is its bonus row), Q rows 0..K_b-1, drafts
0..K_b-1 and uniforms u[b, 0..K_b] (u[b, K_b] is its draw); rows, drafts and uniforms past
those are never read. A draft count outside [0, K] or a negative or non-finite
temperature makes that sequence an error (STATUS_BAD_PARAM).

Early exit (``early_exit_accept``). The same step, reading each sequence's rows in draft
order and stopping at its first rejection; the pages state that acceptance runs between 52%
and 91% (the DeepSeek-V4-Flash drafter card), so most blocks end early. Reading: a
sequence's drafts are inputs and are all checked (a bad id: STATUS_BAD_DRAFT, nothing read);
then for i = 0..K-1 the rows P_i (and Q_i when sampling) are read, a bad one ends the
sequence with STATUS_NONFINITE, and draft i is tested; the walk stops at the first failed
test j. Only when every draft passes is P_K read (bad: STATUS_NONFINITE). Rows after j are
never read, so whatever they hold cannot change the result: on blocks whose rows are all
usable it equals ``speculative_sample_accept`` (``greedy_accept`` at T == 0), with p_draft /
q_draft NaN past j.

Parity pins: every function here is pinned in ``tests/test_oracle_pins.py`` against
things other than itself (exact enumeration of losslessness, sequential greedy
decoding, library inverse-CDF draws, closed-form acceptance rates, chi-square).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

STATUS_BAD_DRAFT = 1      # a draft id outside [0, V)
STATUS_NONFINITE = 2      # a row with NaN / +inf, or with no finite value
STATUS_ZERO_RESIDUAL = 4  # residual mass was 0 after a rejection; drew from p_j instead
STATUS_BAD_PARAM = 16     # mixed batch: a draft count outside [0, K] or a bad temperature


@dataclass
class OracleResult:
    """Per-sequence outcome of one verify call (the pages' ``AcceptResult``)."""

    n_accepted: np.ndarray          # [B] int32, j in [0, K]; the host's n_keep
    tokens: np.ndarray              # [B, K+1] int32: x_0..x_{j-1}, then the drawn token, then -1
    next_token: np.ndarray          # [B] int32: correction (j < K) or bonus (j == K); -1 on error
    status: np.ndarray              # [B] int32 bit flags (STATUS_*)
    p_draft: Optional[np.ndarray] = None   # [B, K] float64 p_i(x_i)
    q_draft: Optional[np.ndarray] = None   # [B, K] float64 q_i(x_i)
    resid_mass: Optional[np.ndarray] = None  # [B] float64: Z_j if j < K, else 1
    accept_margin: Optional[np.ndarray] = None  # [B, K] |u_i - p_i/q_i| (inf where q == 0)
    cdf_margin: Optional[np.ndarray] = None     # [B] distance of u_K to the nearest CDF boundary
    argmax: Optional[np.ndarray] = None         # [B, K+1] greedy row argmax

    def near_boundary(self, eps: float = 1e-6) -> np.ndarray:
        """[B] bool: some decision of this sequence had its uniform within eps of a boundary.

        Only the accept tests that were actually taken (i <= j) and the final inverse-CDF
        draw count.
        """
        B = self.n_accepted.shape[0]
        out = np.zeros(B, dtype=bool)
        if self.accept_margin is None:
            return out
        for b in range(B):
            j = int(self.n_accepted[b])
            K = self.accept_margin.shape[1]
            taken = self.accept_margin[b, : min(j + 1, K)]
            out[b] = bool(np.any(taken < eps)) or bool(self.cdf_margin[b] < eps)
        return out


def _row_is_bad(z: np.ndarray) -> bool:
    """NaN or +inf anywhere, or no finite value at all."""
    return bool(np.isnan(z).any() or np.isposinf(z).any() or not np.isfinite(z).any())


def row_argmax(z: np.ndarray) -> int:
    """a = min{v : z[v] = max_w z[w]}. Float equality treats -0.0 and +0.0 as equal."""
    m = z.max()
    return int(np.flatnonzero(z == m)[0])


def softmax(z: np.ndarray, T: float) -> np.ndarray:
    """softmax(z / T) in float64, max subtracted; -inf entries get probability 0."""
    y = z / T
    y = y - y.max()
    e = np.exp(y)
    return e / e.sum()


def inverse_cdf(w: np.ndarray, u: float):
    """Smallest v with sum_{t<=v} w[t] > u * sum(w), ascending token id.

    Returns (v, margin): margin is the distance, in normalised units, from u to the
    nearer of the two CDF boundaries that bracket v.
    """
    C = np.cumsum(w)
    Z = C[-1]
    target = u * Z
    hits = np.flatnonzero(C > target)
    v = int(hits[0]) if hits.size else int(np.flatnonzero(w > 0)[-1])
    lo = C[v - 1] / Z if v > 0 else 0.0
    hi = C[v] / Z
    return v, float(min(u - lo, hi - u))


def _draw_law(p, q, j):
    """Unnormalised law of the correction / bonus token after j accepted drafts.

    j < K: the residual max(p_j - q_j, 0); if its mass is not positive (only rounding can
    cause that) p_j instead. j == K: the bonus row p_K. Returns (weights, fell_back).
    """
    K = len(q)
    if j < K:
        r = np.maximum(p[j] - q[j], 0.0)
        if r.sum() > 0:
            return r, False
        return p[j], True
    return p[K], False


def draw_law(P_b: np.ndarray, Q_b: np.ndarray, j: int, T: float) -> np.ndarray:
    """The law ``speculative_sample_accept`` draws from for one sequence (P_b: [K+1, V],
    Q_b: [K, V] float64 logits) after j accepted drafts, unnormalised."""
    K = P_b.shape[0] - 1
    p = [softmax(P_b[r], T) for r in range(K + 1)]
    q = [softmax(Q_b[i], T) for i in range(K)]
    return _draw_law(p, q, j)[0]


def cdf_interval(w: np.ndarray, v: int):
    """[C(v-1), C(v)) / Z: the range of u for which the inverse CDF of w returns v."""
    C = np.cumsum(w)
    Z = C[-1]
    return (C[v - 1] / Z if v > 0 else 0.0), C[v] / Z


def greedy_accept(P: np.ndarray, drafts: np.ndarray) -> OracleResult:
    """Greedy block verify.

    P: [B, K+1, V] float64 base logits (row 0 = p_1, row K = bonus); drafts: [B, K] ints.
    a_r = lowest-index argmax of row r; j = first i < K with x_i != a_i, else K; emit
    x_0..x_{j-1} and a_j.
    """
    P = np.asarray(P, dtype=np.float64)
    drafts = np.asarray(drafts)
    B, K1, V = P.shape
    K = K1 - 1
    n = np.zeros(B, dtype=np.int32)
    tokens = np.full((B, K + 1), -1, dtype=np.int32)
    nxt = np.full(B, -1, dtype=np.int32)
    status = np.zeros(B, dtype=np.int32)
    amax = np.full((B, K + 1), -1, dtype=np.int32)
    for b in range(B):
        st = 0
        if K and (np.any(drafts[b] < 0) or np.any(drafts[b] >= V)):
            st |= STATUS_BAD_DRAFT
        if any(_row_is_bad(P[b, r]) for r in range(K + 1)):
            st |= STATUS_NONFINITE
        status[b] = st
        if st:
            continue
        a = [row_argmax(P[b, r]) for r in range(K + 1)]
        amax[b] = a
        j = K
        for i in range(K):
            if int(drafts[b, i]) != a[i]:
                j = i
                break
        n[b] = j
        tokens[b, :j] = drafts[b, :j]
        tokens[b, j] = a[j]
        nxt[b] = a[j]
    return OracleResult(n, tokens, nxt, status, argmax=amax)


def speculative_sample_accept(P: np.ndarray, Q: np.ndarray, drafts: np.ndarray, T: float,
                              u: np.ndarray) -> OracleResult:
    """Lossless rejection-sampling block verify.

    P: [B, K+1, V], Q: [B, K, V] float64 logits; drafts [B, K]; T >= 0; u: [B, K+1] uniforms
    in [0, 1). T == 0 gives exactly ``greedy_accept``.

    For each sequence: p_r = softmax(P_r / T), q_i = softmax(Q_i / T). Walk i = 0..K-1 and
    accept draft x_i iff u_i * q_i(x_i) < p_i(x_i); stop at the first rejection j. If j < K
    draw the correction from r = max(p_j - q_j, 0) with u_K by inverse CDF; else draw the
    bonus token from p_K with u_K.
    """
    if T == 0:
        return greedy_accept(P, drafts)
    if not (T > 0 and np.isfinite(T)):
        raise ValueError("temperature must be finite and >= 0")
    P = np.asarray(P, dtype=np.float64)
    Q = np.asarray(Q, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    drafts = np.asarray(drafts)
    B, K1, V = P.shape
    K = K1 - 1
    n = np.zeros(B, dtype=np.int32)
    tokens = np.full((B, K + 1), -1, dtype=np.int32)
    nxt = np.full(B, -1, dtype=np.int32)
    status = np.zeros(B, dtype=np.int32)
    pd = np.full((B, K), np.nan)
    qd = np.full((B, K), np.nan)
    zm = np.full(B, np.nan)
    am = np.full((B, K), np.inf)
    cm = np.full(B, np.inf)
    for b in range(B):
        st = 0
        if K and (np.any(drafts[b] < 0) or np.any(drafts[b] >= V)):
            st |= STATUS_BAD_DRAFT
        if any(_row_is_bad(P[b, r]) for r in range(K + 1)) or \
                any(_row_is_bad(Q[b, i]) for i in range(K)):
            st |= STATUS_NONFINITE
        if st:
            status[b] = st
            continue
        p = [softmax(P[b, r], T) for r in range(K + 1)]
        q = [softmax(Q[b, i], T) for i in range(K)]
        j = K
        for i in range(K):
            x = int(drafts[b, i])
            pd[b, i], qd[b, i] = p[i][x], q[i][x]
        for i in range(K):
            px, qx = pd[b, i], qd[b, i]
            if qx > 0:
                am[b, i] = abs(u[b, i] - px / qx)
            if not (u[b, i] * qx < px):
                j = i
                break
        r, fell_back = _draw_law(p, q, j)
        if fell_back:
            st |= STATUS_ZERO_RESIDUAL
        zm[b] = r.sum() if (j < K and not fell_back) else (0.0 if fell_back else 1.0)
        v, cm[b] = inverse_cdf(r, float(u[b, K]))
        status[b] = st
        n[b] = j
        tokens[b, :j] = drafts[b, :j]
        tokens[b, j] = v
        nxt[b] = v
    return OracleResult(n, tokens, nxt, status, p_draft=pd, q_draft=qd, resid_mass=zm,
                        accept_margin=am, cdf_margin=cm)


def mixed_accept(P: np.ndarray, Q: Optional[np.ndarray], drafts: np.ndarray,
                 n_drafts: Optional[np.ndarray], temperatures: np.ndarray,
                 u: Optional[np.ndarray]) -> OracleResult:
    """Mixed serving batch: sequence b verifies its first K_b = n_drafts[b] drafts at its
    own temperature T_b = temperatures[b] (0: greedy).

    P: [B, K+1, V], Q: [B, K, V] (may be None when every T_b is 0), drafts [B, K],
    n_drafts [B] or None (every K_b = K), temperatures [B], u: [B, K+1] (may be None when
    every T_b is 0). Sequence b is ``greedy_accept`` or ``speculative_sample_accept`` on
    P[b, :K_b+1], Q[b, :K_b], drafts[b, :K_b], u[b, :K_b+1]; results are laid out as for K
    (tokens [B, K+1], -1 past the drawn token; p_draft / q_draft NaN past K_b).
    """
    P = np.asarray(P, dtype=np.float64)
    drafts = np.asarray(drafts)
    temperatures = np.asarray(temperatures, dtype=np.float64)
    B, K1, V = P.shape
    K = K1 - 1
    nd = np.full(B, K, dtype=np.int64) if n_drafts is None else np.asarray(n_drafts)
    n = np.zeros(B, dtype=np.int32)
    tokens = np.full((B, K + 1), -1, dtype=np.int32)
    nxt = np.full(B, -1, dtype=np.int32)
    status = np.zeros(B, dtype=np.int32)
    pd = np.full((B, K), np.nan)
    qd = np.full((B, K), np.nan)
    zm = np.full(B, np.nan)
    am = np.full((B, K), np.inf)
    cm = np.full(B, np.inf)
    amax = np.full((B, K + 1), -1, dtype=np.int32)
    for b in range(B):
        kb, tb = int(nd[b]), float(temperatures[b])
        if not (0 <= kb <= K) or not (np.isfinite(tb) and tb >= 0):
            status[b] = STATUS_BAD_PARAM
            continue
        Pb = P[b:b + 1, :kb + 1]
        db = drafts[b:b + 1, :kb]
        if tb == 0:
            r = greedy_accept(Pb, db)
            amax[b, :kb + 1] = r.argmax[0]
        else:
            Qb = np.asarray(Q, dtype=np.float64)[b:b + 1, :kb]
            ub = np.asarray(u, dtype=np.float64)[b:b + 1, :kb + 1]
            r = speculative_sample_accept(Pb, Qb, db, tb, ub)
            pd[b, :kb], qd[b, :kb] = r.p_draft[0], r.q_draft[0]
            zm[b] = r.resid_mass[0]
            am[b, :kb] = r.accept_margin[0]
            cm[b] = r.cdf_margin[0]
        n[b], nxt[b], status[b] = r.n_accepted[0], r.next_token[0], r.status[0]
        tokens[b, :kb + 1] = r.tokens[0]
    return OracleResult(n, tokens, nxt, status, p_draft=pd, q_draft=qd, resid_mass=zm,
                        accept_margin=am, cdf_margin=cm, argmax=amax)


def early_exit_accept(P: np.ndarray, Q: Optional[np.ndarray], drafts: np.ndarray, T: float,
                      u: Optional[np.ndarray]) -> OracleResult:
    """The verify step read row by row, stopping each sequence at its first rejection.

    P: [B, K+1, V], Q: [B, K, V] float64 logits (Q and u may be None when T == 0); drafts
    [B, K]; u: [B, K+1]. Sequence b walks i = 0..K-1: P_i (and Q_i) must be usable rows, then
    draft x_i is tested (T == 0: x_i == argmax P_i; else u_i q_i(x_i) < p_i(x_i)); the first
    failure is j. Every draft accepted: P_K must be usable and j = K. The token is argmax P_j
    (T == 0) or the inverse CDF at u_K of max(p_j - q_j, 0) (p_j if that has no mass) or of
    p_K. Rows after j are not looked at.
    """
    greedy = T == 0
    if not greedy and not (T > 0 and np.isfinite(T)):
        raise ValueError("temperature must be finite and >= 0")
    P = np.asarray(P, dtype=np.float64)
    drafts = np.asarray(drafts)
    B, K1, V = P.shape
    K = K1 - 1
    if not greedy:
        Q = np.asarray(Q, dtype=np.float64)
        u = np.asarray(u, dtype=np.float64)
    n = np.zeros(B, dtype=np.int32)
    tokens = np.full((B, K + 1), -1, dtype=np.int32)
    nxt = np.full(B, -1, dtype=np.int32)
    status = np.zeros(B, dtype=np.int32)
    pd = np.full((B, K), np.nan)
    qd = np.full((B, K), np.nan)
    zm = np.full(B, np.nan)
    am = np.full((B, K), np.inf)
    cm = np.full(B, np.inf)
    amax = np.full((B, K + 1), -1, dtype=np.int32)
    for b in range(B):
        if K and (np.any(drafts[b] < 0) or np.any(drafts[b] >= V)):
            status[b] = STATUS_BAD_DRAFT
            continue
        j, bad = K, False
        for i in range(K):
            if _row_is_bad(P[b, i]) or (not greedy and _row_is_bad(Q[b, i])):
                bad = True
                break
            x = int(drafts[b, i])
            if greedy:
                amax[b, i] = row_argmax(P[b, i])
                if x != amax[b, i]:
                    j = i
                    break
            else:
                p, q = softmax(P[b, i], T), softmax(Q[b, i], T)
                pd[b, i], qd[b, i] = p[x], q[x]
                if q[x] > 0:
                    am[b, i] = abs(u[b, i] - p[x] / q[x])
                if not (u[b, i] * q[x] < p[x]):
                    j = i
                    break
        if not bad and j == K and _row_is_bad(P[b, K]):
            bad = True
        if bad:
            status[b] = STATUS_NONFINITE
            pd[b], qd[b], am[b] = np.nan, np.nan, np.inf
            continue
        st = 0
        if greedy:
            v = amax[b, j] = row_argmax(P[b, j])
        else:
            w = softmax(P[b, j], T)
            zm[b] = 1.0
            if j < K:
                r = np.maximum(w - softmax(Q[b, j], T), 0.0)
                if r.sum() > 0:
                    w, zm[b] = r, r.sum()
                else:
                    st, zm[b] = STATUS_ZERO_RESIDUAL, 0.0
            v, cm[b] = inverse_cdf(w, float(u[b, K]))
        status[b] = st
        n[b] = j
        tokens[b, :j] = drafts[b, :j]
        tokens[b, j] = v
        nxt[b] = v
    return OracleResult(n, tokens, nxt, status, p_draft=None if greedy else pd,
                        q_draft=None if greedy else qd, resid_mass=None if greedy else zm,
                        accept_margin=None if greedy else am, cdf_margin=None if greedy else cm,
                        argmax=amax)
