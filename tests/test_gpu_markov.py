"""The Markov-head table mat-vec on the GPU against the float64 oracle.

Tolerance, from the arithmetic. F16, one state: each output is a float32 sum of R = 256
products (8 per lane, then a butterfly), so its error is below (R + 8) 2^-24 sum_k |W[v, k]
h[b, k]|; the tests allow twice R 2^-24 times that sum, plus 1e-30. F16 with two or more states
and Q8_0 with more than ten (tensor cores): the state, scaled by a power of two, is split into
float16 hi + lo within 2^-23 of its largest |h|; the products of the exact table values with
the parts are exact and summed in float32 (F16: one sum per part over all 256 k; Q8_0: per
block of 32, then scaled by d and the 8 blocks added by float32 FMAs). The same 2 R 2^-24
sum |W h| covers the sums; the tests add 2^-22 max_k |h[b, k]| sum_k |W[v, k]| for the split.
One to ten Q8_0 states take exact integer dot products with three signed-byte digit planes of
the state (on the CUDA cores for one state, the integer tensor cores for two to ten), which
represent it within 2^-22 of each block's largest |h| (so within the same added term), then a
few float32 roundings per block.
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
    timeouts = bd.pipeline_timeouts()
    raw = wl.markov_table(V, R, fmt, seed=seed)
    H = wl.markov_states(B, R, seed=seed)
    t = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(DEV)
    y = bd.markov_matvec(t, fmt, torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    W = mk.f16_table(raw) if fmt == "f16" else mk.q8_0_table(raw, R)
    ref = mk.markov_matvec(W, H)
    bound = 2 * R * 2.0 ** -24 * mk.abs_products(W, H) + 1e-30
    hmax = np.abs(H.astype(np.float64)).max(axis=1)                      # [B]
    wsum = np.abs(W).sum(axis=1)                                          # [V]
    bound = bound + 2.0 ** -22 * hmax[:, None] * wsum[None, :]
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= bound), (fmt, V, B, float((err / bound).max()))
    assert bd.pipeline_timeouts() == timeouts


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 7])
def test_serving_vocab(fmt, B):
    _check(129280, B, fmt)


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("B", [5, 7, 10, 11, 16, 17, 48, 64, 65, 130])
def test_many_states(fmt, B):
    """One read of the table per 64 states on the tensor cores (N = 16, 32, 48, 64 and splits)."""
    _check(129280, B, fmt, seed=7)


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("B", [1, 2])
@pytest.mark.parametrize("V", [1, 7, 8, 9, 63, 65, 127, 128, 129, 1000, 262144])
def test_ragged_vocab(fmt, B, V):
    _check(V, B, fmt, seed=5)


@pytest.mark.parametrize("fmt", ["f16", "q8_0"])
@pytest.mark.parametrize("V", [1, 127, 128, 129, 1000, 18943, 262144])
def test_ragged_vocab_tensor_cores(fmt, V):
    """Partial last tiles and grids smaller than the SM count on the tensor-core path."""
    _check(V, 6, fmt, seed=9)


def test_one_hot_state_reads_a_column():
    """h = e_k: y is column k of the table, exactly (one product per output)."""
    V = 4099
    raw = wl.markov_table(V, R, "q8_0", seed=6)
    H = np.zeros((1, R), dtype=np.float32)
    H[0, 77] = 1.0
    y = bd.markov_matvec(torch.from_numpy(raw).to(DEV), "q8_0", torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy()[0].astype(np.float64), mk.q8_0_table(raw, R)[:, 77])



@pytest.mark.parametrize("fmt,B", [("f16", 4), ("q8_0", 3), ("q8_0", 12)])
def test_timeout_path(fmt, B):
    """Each tensor-core kernel (F16; Q8_0 integer; Q8_0 float16) with its first copies withheld:
    the waits for them run out, the kernels give up and free what they hold, the counter grows,
    and the device stays usable: the next normal call is correct."""
    V = 20000
    raw = wl.markov_table(V, R, fmt, seed=10)
    t = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(DEV)
    h = torch.from_numpy(wl.markov_states(B, R, seed=10)).to(DEV)
    before = bd.pipeline_timeouts()
    bd.markov_matvec_withheld(t, fmt, h)
    torch.cuda.synchronize()
    assert bd.pipeline_timeouts() > before
    _check(V, B, fmt, seed=10)
    with pytest.raises(bd.DsparkError):  # one state: the CUDA-core kernels have no waits
        bd.markov_matvec_withheld(t, fmt, h[:1].contiguous())


@pytest.mark.parametrize("fmt,nst", [("f16", 6), ("q8_0", 5), ("q8_0", 9), ("q8_0", 11)])
def test_state_scales(fmt, nst):
    """States of very different magnitudes (each is scaled by its own power of two), a zero
    state and one with a single nonzero entry, in one launch (five Q8_0 states take the
    integer tensor-core kernel (packed and 8-aligned column groups), eleven the float16 one)."""
    V = 5000
    raw = wl.markov_table(V, R, fmt, seed=8)
    H = wl.markov_states(nst, R, seed=8).astype(np.float64)
    H[0] *= 1e-30
    H[1] *= 1e20
    H[2] = 0.0
    H[3] = 0.0
    H[3, 200] = -3.0
    H[4, :128] *= 2.0 ** -140  # subnormal float32 values in half the blocks
    H = H.astype(np.float32)
    t = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(DEV)
    y = bd.markov_matvec(t, fmt, torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    W = mk.f16_table(raw) if fmt == "f16" else mk.q8_0_table(raw, R)
    ref = mk.markov_matvec(W, H)
    bound = 2 * R * 2.0 ** -24 * mk.abs_products(W, H) + \
        2.0 ** -22 * np.abs(H.astype(np.float64)).max(axis=1)[:, None] * np.abs(W).sum(axis=1)[None, :]
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    # subnormal results are flushed by nothing here, but the bound is relative: allow the
    # smallest float32 subnormal on top
    assert np.all(err <= bound + 2.0 ** -149)
    assert np.all(y.cpu().numpy()[2] == 0.0)
    assert np.array_equal(y.cpu().numpy()[3].astype(np.float64), W[:, 200] * -3.0)


@pytest.mark.parametrize("fmt,B", [("f16", 1), ("f16", 4), ("q8_0", 1), ("q8_0", 3), ("q8_0", 7),
                                   ("q8_0", 12)])
def test_nonfinite_states(fmt, B):
    """A state holding a NaN or an infinity gives non-finite results (on every kernel path:
    CUDA cores at one state, the tensor-core kernels above); the other states are unaffected."""
    V = 3000
    raw = wl.markov_table(V, R, fmt, seed=11)
    W = mk.f16_table(raw) if fmt == "f16" else mk.q8_0_table(raw, R)
    H = wl.markov_states(B, R, seed=11)
    bad = 0
    H[bad, 5] = np.nan if B % 2 else np.inf
    t = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(DEV)
    y = bd.markov_matvec(t, fmt, torch.from_numpy(H).to(DEV))
    torch.cuda.synchronize()
    y = y.cpu().numpy().astype(np.float64)
    assert not np.isfinite(y[bad]).any()
    if B > 1:
        good = H[1:]
        ref = mk.markov_matvec(W, good)
        bound = 2 * R * 2.0 ** -24 * mk.abs_products(W, good) + 1e-30 + \
            2.0 ** -22 * np.abs(good.astype(np.float64)).max(axis=1)[:, None] * np.abs(W).sum(axis=1)[None, :]
        assert np.all(np.abs(y[1:] - ref) <= bound)
