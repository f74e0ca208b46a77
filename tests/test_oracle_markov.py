"""Pins of the oracle's Markov-head table mat-vec (``oracle/markov_ref.py``).

The Q8_0 block decoding is checked against a block worked by hand (tests/golden); the
mat-vec against a plain triple loop, a one-hot state and an identity table; the synthetic
Q8_0 tables against the block quantiser's error bound.
"""

import os

import numpy as np

from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import markov_ref as mk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q8_0_block.txt")


def _golden():
    kv = {}
    for line in open(GOLDEN):
        if line.startswith("#") or ":" not in line:
            continue
        k, v = line.split(":", 1)
        kv[k.strip()] = v.split()
    raw = np.array([int(t, 16) for t in kv["bytes"]], dtype=np.uint8)
    return raw, np.array([float(t) for t in kv["values"]])


def test_q8_0_block_worked_by_hand():
    raw, values = _golden()
    assert raw.size == mk.Q8_0_BLOCK_BYTES
    # the same block as the 5th of 8 in a 256-wide row: only its slice takes these values
    row = np.zeros((1, 8 * mk.Q8_0_BLOCK_BYTES), dtype=np.uint8)
    row[0, 4 * 34:5 * 34] = raw
    got = mk.q8_0_table(row, 256)
    assert np.array_equal(got[0, 128:160], values)
    assert np.all(got[0, :128] == 0) and np.all(got[0, 160:] == 0)


def test_f16_values_are_exact():
    bits = np.array([[0x3C00, 0xC000, 0x3800, 0x0001, 0x7BFF, 0x8000]], dtype=np.uint16)
    assert np.array_equal(mk.f16_table(bits)[0], [1.0, -2.0, 0.5, 2.0 ** -24, 65504.0, 0.0])


def test_matvec_equals_a_triple_loop():
    rng = np.random.default_rng(3)
    W = rng.normal(size=(9, 5))
    H = rng.normal(size=(3, 5))
    want = np.zeros((3, 9))
    for b in range(3):
        for v in range(9):
            acc = 0.0
            for k in range(5):
                acc += W[v, k] * H[b, k]
            want[b, v] = acc
    assert np.allclose(mk.markov_matvec(W, H), want, rtol=1e-14, atol=1e-14)


def test_one_hot_state_and_identity_table():
    rng = np.random.default_rng(4)
    W = rng.normal(size=(40, 8))
    H = np.zeros((1, 8))
    H[0, 3] = 1.0
    assert np.array_equal(mk.markov_matvec(W, H)[0], W[:, 3])       # column of the table
    H = rng.normal(size=(2, 8))
    assert np.array_equal(mk.markov_matvec(np.eye(8), H), H)       # rows are unit vectors


def test_synthetic_q8_0_table_within_the_quantiser_bound():
    """The generator's blocks decode to within half a quantum of the float values."""
    V, R = 50, 256
    raw = wl.markov_table(V, R, "q8_0")
    assert raw.shape == (V, R // 32 * 34)
    got = mk.q8_0_table(raw, R)
    ref = mk.f16_table(wl.markov_table(V, R, "f16"))   # the same values, rounded to half
    d = np.abs(got).reshape(V, R // 32, 32).max(axis=2) / 127.0
    err = np.abs(got - ref).reshape(V, R // 32, 32)
    assert np.all(err <= (d[:, :, None] * 0.5 * 1.01 + np.abs(ref).reshape(V, R // 32, 32) * 2e-3))



def test_table_sizes_match_the_card():
    """The drafter card says the Q8_0 form of markov_w2 makes the file 31 MB smaller than the
    F16 form. With the reading V = 129280 rows (the drafter's vocabulary) of R = 256 values,
    2 bytes each in F16 and 34 bytes per 32 values in Q8_0, the two tables differ by 31.0 MB."""
    V, R = 129280, 256
    f16 = wl.markov_table(8, R, "f16").shape[1] * 2 * V
    q8 = wl.markov_table(8, R, "q8_0").shape[1] * V
    assert q8 == V * (R // 32) * mk.Q8_0_BLOCK_BYTES
    assert round((f16 - q8) / 1e6) == 31


def _matrix(text):
    return np.asarray([[float(x) for x in row.split()] for row in text.split(";")])


def test_abs_products_worked_by_hand():
    """The error scale that sets the GPU test's tolerance, on a 2 x 2 case worked by hand
    (tests/golden/abs_products_2x2.txt): a transposed operand or a dropped absolute value
    changes the result."""
    kv = {}
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "abs_products_2x2.txt")):
        if line.strip() and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = _matrix(v)
    got = mk.abs_products(kv["W"], kv["h"])
    assert np.array_equal(got, kv["abs_products"])
    assert not np.array_equal(mk.markov_matvec(kv["W"], kv["h"]), kv["abs_products"])
