"""The FMA-pipe 2^x of the kernels (common.cuh ``exp2_poly``), evaluated on the CPU in
float32 with its coefficients read from the source: as accurate as the SFU's ex2.approx
(relative error within 2 ulp) on the range the kernels use, exact at 0, 0 below 2^-125."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "lossless_draft_verification_speculative_b200", "csrc")
sys.path.insert(0, CSRC)

import gen_exp2_poly as gen  # noqa: E402


def device_coefficients():
    src = open(os.path.join(CSRC, "common.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"__int_as_float\((0x[0-9a-f]{8})\)", body)
    c = [np.uint32(int(h, 16)).view(np.float32) for h in hexes]  # c5, c4, c3, c2, c1
    assert len(c) == 5 and "__fmaf_rn(p, f, 1.f)" in body
    return [np.float32(1.0)] + c[::-1]


def test_device_constants_are_the_generators():
    dev = device_coefficients()
    fit = gen.fit()
    assert [float(a) for a in dev] == [float(b) for b in fit]


def test_relative_error_within_two_ulp():
    coef = device_coefficients()
    x = np.concatenate([np.random.default_rng(7).uniform(-125.0, 0.0, 400_000),
                        -np.abs(np.random.default_rng(8).normal(0.0, 1e-3, 100_000)),
                        -np.arange(0, 126, dtype=np.float64)]).astype(np.float32)
    y = gen.eval_f32(coef, x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 2 * 2.0 ** -23
    assert gen.eval_f32(coef, np.array([0.0], np.float32))[0] == 1.0
    # integer exponents are exact powers of two
    k = -np.arange(0, 126, dtype=np.float32)
    assert np.array_equal(gen.eval_f32(coef, k), np.exp2(k).astype(np.float32))
