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


def to_dev(arr, dtype):
    arr = np.ascontiguousarray(arr)
    if dtype == "bf16":
        return torch.from_numpy(arr.view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(arr.astype(np.float32)).to(DEV)


def run_gpu(P, Q, d, u, T, dtype, block=None):
    """One verify call through the binding. P: [B, K+1, V] stored logits (or a (p1, pv) pair
    of device tensors via ``block``). Returns host numpy arrays."""
    Pd = block if block is not None else to_dev(P, dtype)
    K = d.shape[1]
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    if T == 0:
        r = bd.greedy_accept(Pd, dd)
    else:
        Qd = to_dev(Q, dtype) if K > 0 else None
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


def compare_sampling(g, o, label=""):
    """Tolerances of the sampling policy. Returns the number of near-boundary sequences.

    p_i(x_i), q_i(x_i) and the residual mass within PROB_RTOL relative; accepted count and
    tokens identical except for sequences where a uniform lies within BOUNDARY_EPS of an
    accept-test or inverse-CDF boundary (those are counted, not compared).
    """
    assert np.array_equal(g["status"] & ERR_BITS, o.status & ERR_BITS), label
    ok = (o.status & ERR_BITS) == 0
    near = o.near_boundary(BOUNDARY_EPS) & ok
    same = ok & ~near
    bad = np.flatnonzero(same & ((g["n_accepted"] != o.n_accepted) |
                                 np.any(g["tokens"] != o.tokens, axis=1)))
    assert bad.size == 0, (label, bad[:10], g["n_accepted"][bad[:10]], o.n_accepted[bad[:10]],
                           g["tokens"][bad[:3]], o.tokens[bad[:3]])
    err = ~ok
    assert np.all(g["n_accepted"][err] == 0) and np.all(g["next_token"][err] == -1)
    K = g["tokens"].shape[1] - 1
    if K:
        for key, ref in (("p_draft", o.p_draft), ("q_draft", o.q_draft)):
            gv, ov = g[key][ok].astype(np.float64), ref[ok]
            np.testing.assert_allclose(gv, ov, rtol=PROB_RTOL, atol=1e-37, err_msg=label + key)
        rej = same & (o.n_accepted < K) & ((o.status & bd.SEQ_ZERO_RESIDUAL) == 0)
        np.testing.assert_allclose(g["resid_mass"][rej].astype(np.float64), o.resid_mass[rej],
                                   rtol=PROB_RTOL, atol=RESID_ATOL, err_msg=label + "resid_mass")
    return int(near.sum())
