"""Coefficients of the FMA-pipe 2^x of the verify kernels (``exp2_poly`` in common.cuh).

2^x is split as 2^n * 2^f with n = rint(x), |f| <= 1/2. On that interval 2^f is replaced by
p(f) = 1 + c1 f + ... + c5 f^5, fitted here by least squares on Chebyshev nodes with the
weights iterated toward the minimax of the relative error (p(0) = 1 is kept exact). The script
prints the coefficients as float32 and the error of the whole reduction evaluated in float32
fused multiply-adds on random x in [-125, 0]:

    python gen_exp2_poly.py
"""

import numpy as np

DEG = 5


def fit(deg: int = DEG):
    xs = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    w = np.ones_like(xs)
    for _ in range(80):
        A = np.vander(xs, deg + 1, increasing=True)[:, 1:] / (2.0 ** xs)[:, None]
        rhs = 1.0 - 1.0 / (2.0 ** xs)
        c, *_ = np.linalg.lstsq(A * w[:, None], w * rhs, rcond=None)
        err = np.abs(A @ c - rhs)
        w = w * (1.0 + err / err.max()) ** 2
        w /= w.mean()
    return [np.float32(1.0)] + [np.float32(v) for v in c]


def eval_f32(coef, x):
    """The device reduction in float32: rint by the 1.5*2^23 shift, Horner in FMAs (a*b is
    exact in float64, one rounding to float32 per step), n added to the exponent bits."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full(f.shape, coef[-1], dtype=np.float32)
    for c in coef[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    return (p.view(np.int32) + (n.astype(np.int32) << 23)).view(np.float32)


if __name__ == "__main__":
    coef = fit()
    x = np.random.default_rng(1).uniform(-125.0, 0.0, 1_000_000).astype(np.float32)
    rel = eval_f32(coef, x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0
    for k, c in enumerate(coef):
        print(f"c{k} = {float(c):.9e}f  // {hex(c.view(np.uint32))}")
    print(f"max |relative error| {np.abs(rel).max():.3e}, mean {rel.mean():.2e}")
