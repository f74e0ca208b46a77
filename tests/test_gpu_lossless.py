"""Exact losslessness of the CUDA path at V=4, K=2, by enumeration.

The same enumeration that pins the oracle (tests/enumeration.py) runs the GPU's sampling
verify on every (draft tuple, uniform cell) pair of the Farey grid: rows with probabilities
in eighths (quarters at T != 1), every uniform coordinate at the midpoint of an interval
between consecutive members of F_denom. Every accept ratio and every normalised CDF point
lies in F_denom, and a midpoint is at least 1/(2 denom^2) - 2^-25 away from all of them, far
beyond float32 rounding of the logits and the GPU's float32 arithmetic, so the GPU must return
the oracle's tokens on every cell, and the emitted law computed from its results must equal
p_1 x p_2 x p_3 exactly (dspark-mlx wheel adapter.py docstring, "lossless accept policy";
DeepSeek-V4-Flash DSpark drafter card, "lossless by construction").
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd

import enumeration as en

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
F8 = lambda *xs: [Fraction(x, 8) for x in xs]  # noqa: E731
F4 = lambda *xs: [Fraction(x, 4) for x in xs]  # noqa: E731


def _gpu_runner(zP, zQ, d, T, u):
    """The sampling verify through the binding on float32 logits (-inf kept)."""
    P = torch.from_numpy(zP.astype(np.float32)).to(DEV)
    Q = torch.from_numpy(zQ.astype(np.float32)).to(DEV)
    dd = torch.from_numpy(d.astype(np.int32)).to(DEV)
    ud = torch.from_numpy(u.astype(np.float32)).to(DEV)
    r = bd.speculative_sample_accept(P, Q, dd, T, ud)
    torch.cuda.synchronize()
    assert int(r.status.abs().sum()) == 0
    return type("GpuResult", (), {"n_accepted": r.n_accepted.cpu().numpy(),
                                  "tokens": r.tokens.cpu().numpy()})


CASES = [
    ("eighths", [F8(4, 2, 1, 1), F8(1, 1, 2, 4), F8(2, 2, 3, 1)],
     [F8(2, 3, 2, 1), F8(4, 2, 1, 1)], 1.0, 8),
    ("masked", [F8(0, 4, 4, 0), F8(1, 0, 3, 4), F8(0, 0, 0, 8)],
     [F8(2, 2, 2, 2), F8(0, 4, 0, 4)], 1.0, 8),
    ("quarters_T0.5", [F4(2, 1, 1, 0), F4(0, 1, 1, 2), F4(1, 1, 1, 1)],
     [F4(1, 1, 1, 1), F4(2, 2, 0, 0)], 0.5, 4),
    ("quarters_T2", [F4(2, 1, 1, 0), F4(0, 1, 1, 2), F4(1, 1, 1, 1)],
     [F4(1, 1, 1, 1), F4(2, 2, 0, 0)], 2.0, 4),
]


@pytest.mark.parametrize("name,Pp,Qp,T,denom", CASES, ids=[c[0] for c in CASES])
def test_gpu_emitted_law_is_exactly_the_target(name, Pp, Qp, T, denom):
    law_gpu, res_gpu = en.enumerate_emitted(Pp, Qp, T, denom, runner=_gpu_runner)
    law_ora, res_ora = en.enumerate_emitted(Pp, Qp, T, denom)
    # token for token on every cell of the grid
    assert np.array_equal(res_gpu.n_accepted, res_ora.n_accepted)
    assert np.array_equal(res_gpu.tokens, res_ora.tokens)
    # and therefore the exact law
    assert law_gpu == en.product_dist(Pp)
    assert law_gpu == law_ora
