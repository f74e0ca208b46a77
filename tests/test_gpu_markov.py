"""The Markov-head table mat-vec on the GPU against the float64 oracle.

Tolerance, from the arithmetic: each output is a float32 sum of R = 256 products (8 per
lane, then a butterfly; or 32 per Q8_0 block, a scale multiply, then 8 blocks), so its error
is below (R + 8) * 2^-24 * sum_k |W[v, k] h[b, k]|; the tests allow twice R * 2^-24 times that
sum, plus 1e-30.
"""

import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import markov_ref as mk

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
R = 256


def _check(V, B, fmt, seed=4):
    raw = wl.markov_table(V, R, fmt, seed=seed)
    H = wl.markov_states(B, R, seed=seed)
    t = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(DEV)
    y = bd.markov_matvec(t, fmt, torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    W = mk.f16_table(raw) if fmt == "f16" else mk.q8_0_table(raw, R)
    ref = mk.markov_matvec(W, H)
    bound = 2 * R * 2.0 ** -24 * mk.abs_products(W, H) + 1e-30
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= bound), (fmt, V, B, float((err / bound).max()))


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 7])
def test_serving_vocab(fmt, B):
    _check(129280, B, fmt)


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("V", [1, 7, 8, 9, 63, 65, 1000, 262144])
def test_ragged_vocab(fmt, V):
    _check(V, 2, fmt, seed=5)


def test_one_hot_state_reads_a_column():
    """h = e_k: y is column k of the table, exactly (one product per output)."""
    V = 4099
    raw = wl.markov_table(V, R, "q8_0", seed=6)
    H = np.zeros((1, R), dtype=np.float32)
    H[0, 77] = 1.0
    y = bd.markov_matvec(torch.from_numpy(raw).to(DEV), "q8_0", torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy()[0].astype(np.float64), mk.q8_0_table(raw, R)[:, 77])

