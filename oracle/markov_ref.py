"""CPU float64 oracle of the drafter's Markov-head table mat-vec.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
arms may import or run this module; the product path never does.

What it computes. The DSpark drafter adds a previous-token correction through a rank-256
Markov head (mlx-dspark README, "How it works"); its second table, ``markov_w2``, maps the
rank-R state to one bias per vocabulary entry, and the ds4 engine reads that table in full
four times per draft block as a mat-vec (the DeepSeek-V4-Flash DSpark drafter card, "Files":
0.18 ms per call with the table in Q8_0 instead of 0.63 ms in F16 on a GB10). Reading: with
W the table as V rows of R values (row v holds vocab entry v's R coordinates, contiguous, as
GGUF stores a weight whose ne[0] is R) and h_b a rank-R state,

    y[b, v] = sum_k W[v, k] * h[b, k].

Storage forms, both named by the card: F16, V x R half floats; Q8_0, the GGUF block format:
each row is R/32 blocks of 34 bytes, a little-endian float16 scale d then 32 signed bytes q,
and the value of element i of the block is d * q[i].
"""

from __future__ import annotations

import numpy as np

QK8_0 = 32                 # values per Q8_0 block
Q8_0_BLOCK_BYTES = 2 + QK8_0


def f16_table(raw: np.ndarray) -> np.ndarray:
    """[V, R] uint16 half-float bit patterns -> exact float64 values."""
    return np.asarray(raw, dtype=np.uint16).view(np.float16).astype(np.float64)


def q8_0_table(raw: np.ndarray, R: int) -> np.ndarray:
    """[V, R/32 * 34] uint8 rows of Q8_0 blocks -> float64 [V, R] values d * q (exact: the
    product of a half and a small integer fits a double)."""
    raw = np.asarray(raw, dtype=np.uint8)
    V = raw.shape[0]
    nb = R // QK8_0
    blocks = raw.reshape(V, nb, Q8_0_BLOCK_BYTES)
    d = blocks[:, :, 0:2].copy().view("<f2")[:, :, 0].astype(np.float64)   # [V, nb]
    q = blocks[:, :, 2:].view(np.int8).astype(np.float64)                   # [V, nb, 32]
    return (q * d[:, :, None]).reshape(V, R)


def markov_matvec(W: np.ndarray, H: np.ndarray) -> np.ndarray:
    """y[b, v] = sum_k W[v, k] h[b, k] in float64. W: [V, R] values, H: [B, R] -> [B, V]."""
    W = np.asarray(W, dtype=np.float64)
    H = np.asarray(H, dtype=np.float64)
    return H @ W.T


def abs_products(W: np.ndarray, H: np.ndarray) -> np.ndarray:
    """sum_k |W[v, k] h[b, k]| [B, V]: the scale of the rounding error of a float32 sum."""
    return np.abs(np.asarray(H, dtype=np.float64)) @ np.abs(np.asarray(W, dtype=np.float64)).T
