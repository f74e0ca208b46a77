"""Shared helpers of the GPU tests: run the CUDA path through the C ABI, compare to the oracle."""

import numpy as np
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import accept_ref as ora

DEV = "cuda:0"
PROB_RTOL = 1e-5        # probabilities: fp32 accumulate vs fp64
BOUNDARY_EPS = 1e-6     # decisions may differ only where u is this close to a boundary
# The residual mass sum_v max(p - q, 0) cancels: each fp32 p[v], q[v] carries a few ulp of
# relative error (<= ~5e-7), so the absolute error of the sum is bounded by about
# 5e-7 * (sum p + sum q) = 1e-6 whatever Z is. Relative 1e-5 plus this absolute floor.
RESID_ATOL = 2e-6
ERR_BITS = bd.SEQ_BAD_DRAFT | bd.SEQ_NONFINITE

# (label, sequences compared, near-boundary sequences, of which the GPU result differed):
# every sampling comparison of the run, printed in the session summary (conftest.py)
NEAR_LOG = []


def to_dev(arr, dtype):
    arr = np.ascontiguousarray(arr)
    if dtype == "bf16":
        return torch.from_numpy(arr.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(arr.astype(np.float32)).to(DEV)


def run_gpu(P, Q, d, u, T, dtype, block=None, Q_dev=None):
    """One verify call through the binding. P: [B, K+1, V] stored logits (or a device block /
    (p1, pv) pair via ``block``; ``Q_dev``: Q already on the device). Returns host numpy
    arrays."""
    Pd = block if block is not None else to_dev(P, dtype)
    K = d.shape[1]
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    if T == 0:
        r = bd.greedy_accept(Pd, dd)
    else:
        Qd = Q_dev if Q_dev is not None else (to_dev(Q, dtype) if K > 0 else None)
        r = bd.speculative_sample_accept(Pd, Qd, dd, T, ud)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in vars(r).items() if v is not None}


def run_oracle(P, Q, d, u, T, dtype):
    Pf = wl.as_float64(P, dtype)
    if T == 0:
        return ora.greedy_accept(Pf, d)
    return ora.speculative_sample_accept(Pf, wl.as_float64(Q, dtype), d, T, u.astype(np.float64))


def compare_greedy(g, o):
    """Bit-exact: accepted count, tokens, next token and error bits."""
    assert np.array_equal(g["n_accepted"], o.n_accepted)
    assert np.array_equal(g["tokens"], o.tokens)
    assert np.array_equal(g["next_token"], o.next_token)
    assert np.array_equal(g["status"] & ERR_BITS, o.status & ERR_BITS)


def compare_sampling(g, o, label="", inputs=None):
    """Tolerances of the sampling policy. Returns the number of near-boundary sequences.

    p_i(x_i), q_i(x_i) within PROB_RTOL relative, the residual mass within PROB_RTOL plus
    RESID_ATOL. Accepted count and tokens identical, except where a uniform lies within
    BOUNDARY_EPS of a boundary; those sequences are counted and checked for what they are:
    a differing accept decision must have |u_i - p_i/q_i| < BOUNDARY_EPS in the oracle, and a
    differing drawn token must have u_K within BOUNDARY_EPS of that token's interval of the
    oracle's float64 CDF. ``inputs`` = (P, Q, u, T, dtype) enables the token check.
    """
    assert np.array_equal(g["status"] & ERR_BITS, o.status & ERR_BITS), label
    ok = (o.status & ERR_BITS) == 0
    err = ~ok
    assert np.all(g["n_accepted"][err] == 0) and np.all(g["next_token"][err] == -1)
    K = g["tokens"].shape[1] - 1
    near = 0
    flagged = int(np.count_nonzero(o.near_boundary(BOUNDARY_EPS)[ok])) \
        if o.accept_margin is not None else 0
    for b in np.flatnonzero(ok):
        jg, jo = int(g["n_accepted"][b]), int(o.n_accepted[b])
        if jg != jo:
            k = min(jg, jo)
            assert o.accept_margin[b, k] < BOUNDARY_EPS, (label, b, jg, jo, o.accept_margin[b])
            near += 1
            continue
        assert np.array_equal(g["tokens"][b, :jg], o.tokens[b, :jo]), (label, b)
        tg, to = int(g["tokens"][b, jg]), int(o.tokens[b, jo])
        if tg != to:
            assert inputs is not None, (label, b, tg, to)
            P, Q, u, T, dtype = inputs
            w = ora.draw_law(wl.as_float64(P[b], dtype), wl.as_float64(Q[b], dtype), jg, T)
            assert 0 <= tg < w.shape[0] and w[tg] > 0, (label, b, tg)
            lo, hi = ora.cdf_interval(w, tg)
            uK = float(u[b, K])
            assert lo - BOUNDARY_EPS <= uK < hi + BOUNDARY_EPS, (label, b, tg, to, lo, hi, uK)
            near += 1
        assert np.all(g["tokens"][b, jg + 1:] == -1)
    if K:
        for key, ref in (("p_draft", o.p_draft), ("q_draft", o.q_draft)):
            gv, ov = g[key][ok].astype(np.float64), ref[ok]
            np.testing.assert_allclose(gv, ov, rtol=PROB_RTOL, atol=1e-37, err_msg=label + key)
        rej = ok & (o.n_accepted < K) & (g["n_accepted"] == o.n_accepted) & \
            ((o.status & bd.SEQ_ZERO_RESIDUAL) == 0)
        np.testing.assert_allclose(g["resid_mass"][rej].astype(np.float64), o.resid_mass[rej],
                                   rtol=PROB_RTOL, atol=RESID_ATOL, err_msg=label + "resid_mass")
    NEAR_LOG.append((label, int(np.count_nonzero(ok)), flagged, near))
    return near
