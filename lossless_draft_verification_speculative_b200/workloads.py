"""Seeded synthetic verify-block inputs: base logits P, draft logits Q, drafts, uniforms.

This module only *makes inputs*. It holds none of the verify/accept arithmetic: no
softmax, no acceptance test, no residual and no inverse-CDF draw. Drafts are drawn
the way a drafter would draw them, from softmax(Q/T), but through the Gumbel-max
identity (argmax of Q/T plus i.i.d. Gumbel noise), so no probability is ever formed
here. Both the CPU oracle's tests and the CUDA path's tests/bench take their inputs
from here, so the two sides see bit-identical logits, drafts and uniforms.

Shapes follow the block convention of the dspark-mlx wheel (page "dspark-mlx
0.1.0__py3-none-any.whl", ``dspark_mlx/adapter.py`` module docstring, "Logit
conventions"): row 0 of P is p_1 from the anchor step, rows 1..K are p_2..p_{K+1}
from the verify forward (row K is the bonus position), and Q holds the K draft rows.

Every sequence b draws from its own generator ``default_rng([seed, b, ...])``, so any
subset of sequences can be regenerated on its own (the oracle checks sampled
sequences of the large workloads without materialising the whole batch twice).

Readings of the workload descriptions: "N(0, s)" names a standard deviation; values are generated in float32 and
rounded to bf16 with round-to-nearest-even; drafts are drawn from the *rounded* Q
that the verifier will see.
"""

from __future__ import annotations

import os
from dataclasses import dataclass, field
from typing import Iterable, Optional, Sequence

import numpy as np

SEED_LOGITS = 0
SEED_DRAFTS = 1
SEED_UNIFORMS = 2


@dataclass(frozen=True)
class Workload:
    """One synthetic verify workload: B sequences, K drafts each, vocabulary V."""

    name: str
    B: int
    K: int
    V: int
    dtype: str                      # "f32" or "bf16": storage type of P and Q
    kind: str                       # logit recipe, see ``_row_logits``
    temperatures: tuple = (1.0,)
    cycles: int = 1                 # verify cycles the description asks for
    description: str = ""
    params: dict = field(default_factory=dict)

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def sampling_bytes(self) -> int:
        """Algorithmic bytes of one sampling verify: every P and Q element read once."""
        return self.elem_bytes * self.V * self.B * (2 * self.K + 1)

    def greedy_bytes(self) -> int:
        """Algorithmic bytes of one greedy verify: every P element read once."""
        return self.elem_bytes * self.V * self.B * (self.K + 1)


WORKLOADS = {
    "tiny": Workload(
        "tiny", B=1, K=3, V=64, dtype="f32", kind="iid", temperatures=(1.0,), cycles=1000,
        description="B1 K3 V64 fp32, P and Q i.i.d. N(0,2), drafts ~ softmax(Q), T=1",
        params={"sd": 2.0}),
    "qwen3_4b_block7": Workload(
        "qwen3_4b_block7", B=1, K=7, V=151936, dtype="bf16", kind="shared_noise",
        temperatures=(1.0, 0.0), cycles=10000,
        description="B1 K7 V151936 bf16, z~N(0,3), Q = z + N(0,1)",
        params={"sd": 3.0, "noise": 1.0}),
    "gemma4_12b_block7": Workload(
        "gemma4_12b_block7", B=8, K=7, V=262144, dtype="bf16", kind="softcap",
        temperatures=(1.0, 0.0),
        description="B8 K7 V262144 bf16, P = 30 tanh(z/30), z~N(0,4), Q = 30 tanh((z+N(0,0.5))/30)",
        params={"sd": 4.0, "noise": 0.5, "cap": 30.0}),
    "dsv4_flash_serving": Workload(
        "dsv4_flash_serving", B=64, K=7, V=129280, dtype="bf16", kind="mixed_sigma",
        temperatures=(0.0, 0.7, 1.0),
        description="B64 K7 V129280 bf16, z~N(0,3), Q = z + N(0,sigma_b), sigma_b in {0.25,1,4}",
        params={"sd": 3.0, "sigmas": (0.25, 1.0, 4.0)}),
    "stress": Workload(
        "stress", B=256, K=15, V=262144, dtype="bf16", kind="zipf",
        temperatures=(0.0, 0.6, 1.0),
        description="B256 K15 V262144 bf16, logit = -1.1 ln(rank) + N(0,0.5) over a random "
                    "vocab permutation per row, Q = same + N(0,1)",
        params={"slope": 1.1, "sd": 0.5, "noise": 1.0}),
}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Inputs here are always finite, so no NaN special case is needed.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact: bf16 is the top half of a float32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def _row_logits(w: Workload, b: int, seed: int):
    """float32 P [K+1, V] and Q [K, V] of sequence b, before storage rounding."""
    rng = _rng(seed, b)
    K, V, p = w.K, w.V, w.params
    if w.kind == "iid":
        P = rng.normal(0.0, p["sd"], size=(K + 1, V)).astype(np.float32)
        Q = rng.normal(0.0, p["sd"], size=(K, V)).astype(np.float32)
    elif w.kind == "shared_noise":
        z = rng.normal(0.0, p["sd"], size=(K + 1, V)).astype(np.float32)
        P = z
        Q = (z[:K] + rng.normal(0.0, p["noise"], size=(K, V))).astype(np.float32)
    elif w.kind == "softcap":
        cap = p["cap"]
        z = rng.normal(0.0, p["sd"], size=(K + 1, V))
        P = (cap * np.tanh(z / cap)).astype(np.float32)
        Q = (cap * np.tanh((z[:K] + rng.normal(0.0, p["noise"], size=(K, V))) / cap)).astype(np.float32)
    elif w.kind == "mixed_sigma":
        sigma = float(rng.choice(np.asarray(p["sigmas"], dtype=np.float64)))
        z = rng.normal(0.0, p["sd"], size=(K + 1, V)).astype(np.float32)
        P = z
        Q = (z[:K] + rng.normal(0.0, sigma, size=(K, V))).astype(np.float32)
    elif w.kind == "zipf":
        base = -p["slope"] * np.log(np.arange(1, V + 1, dtype=np.float64))
        perm = rng.permuted(np.tile(np.arange(V), (K + 1, 1)), axis=1)
        P = (base[perm] + rng.normal(0.0, p["sd"], size=(K + 1, V))).astype(np.float32)
        Q = (P[:K] + rng.normal(0.0, p["noise"], size=(K, V))).astype(np.float32)
    else:
        raise ValueError(f"unknown logit recipe {w.kind!r}")
    return P, Q


def sequence_sigma(w: Workload, b: int, seed: int = SEED_LOGITS) -> Optional[float]:
    """The draft-noise standard deviation drawn for sequence b (mixed_sigma only)."""
    if w.kind != "mixed_sigma":
        return None
    rng = _rng(seed, b)
    return float(rng.choice(np.asarray(w.params["sigmas"], dtype=np.float64)))


def logits(w: Workload, seqs: Optional[Iterable[int]] = None, seed: int = SEED_LOGITS):
    """Stored P [n, K+1, V] and Q [n, K, V] for sequences ``seqs`` (default: all B).

    bf16 workloads return uint16 bit patterns, f32 workloads return float32.
    """
    seqs = list(range(w.B)) if seqs is None else list(seqs)
    store = np.float32 if w.dtype == "f32" else np.uint16
    P = np.empty((len(seqs), w.K + 1, w.V), dtype=store)
    Q = np.empty((len(seqs), w.K, w.V), dtype=store)
    for n, b in enumerate(seqs):
        p, q = _row_logits(w, b, seed)
        if w.dtype == "f32":
            P[n], Q[n] = p, q
        else:
            P[n], Q[n] = round_to_bf16_bits(p), round_to_bf16_bits(q)
    return P, Q


def as_float64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of stored logits (bf16 bits or float32)."""
    if dtype == "f32":
        return np.asarray(stored, dtype=np.float32).astype(np.float64)
    return bf16_bits_to_f32(stored).astype(np.float64)


def drafts(w: Workload, Q_stored: np.ndarray, T: float, seqs: Optional[Sequence[int]] = None,
           seed: int = SEED_DRAFTS, cycle: int = 0) -> np.ndarray:
    """Draft tokens [n, K] int32 drawn from softmax(Q/T) of the stored Q, as a drafter does.

    T > 0: Gumbel-max, argmax_v (Q[v]/T + G_v) with G_v i.i.d. standard Gumbel, which is an
    exact draw from softmax(Q/T). T == 0: the drafter's greedy pick, argmax_v Q[v].
    """
    n = Q_stored.shape[0]
    seqs = list(range(n)) if seqs is None else list(seqs)
    Qf = as_float64(Q_stored, w.dtype)
    out = np.empty((n, w.K), dtype=np.int32)
    t_key = int(round(T * 1000))
    for k, b in enumerate(seqs):
        if T == 0:
            out[k] = np.argmax(Qf[k], axis=-1)
            continue
        rng = _rng(seed, b, t_key, cycle)
        u = rng.random(size=(w.K, w.V))
        g = -np.log(-np.log(np.maximum(u, np.finfo(np.float64).tiny)))
        out[k] = np.argmax(Qf[k] / T + g, axis=-1)
    return out


def uniforms(w: Workload, seqs: Optional[Sequence[int]] = None, T: float = 1.0,
             seed: int = SEED_UNIFORMS, cycle: int = 0) -> np.ndarray:
    """Per-sequence uniforms [n, K+1] float32 in [0, 1): u[b, i] tests draft i, u[b, K] is
    the one draw used for the resample or the bonus token."""
    seqs = list(range(w.B)) if seqs is None else list(seqs)
    t_key = int(round(T * 1000))
    out = np.empty((len(seqs), w.K + 1), dtype=np.float32)
    for k, b in enumerate(seqs):
        out[k] = _rng(seed, b, t_key, cycle).random(size=w.K + 1, dtype=np.float32)
    return out


SEED_MIXED = 3


def mixed_params(w: Workload, temperatures: Sequence[float] = (0.0, 0.7, 1.0),
                 seed: int = SEED_MIXED):
    """Per-sequence draft counts K_b [B] int32 and temperatures T_b [B] float32 of a mixed
    serving batch: K_b = K for 40% of the sequences (a full block), else uniform on 0..K-1
    (a block truncated by a confidence threshold or a cap); T_b uniform on ``temperatures``."""
    rng = _rng(seed, w.B, w.K)
    full = rng.random(w.B) < 0.4
    kb = np.where(full, w.K, rng.integers(0, max(w.K, 1), size=w.B)).astype(np.int32)
    T = np.asarray(temperatures, dtype=np.float32)[rng.integers(0, len(temperatures), size=w.B)]
    return kb, T


def mixed_inputs(w: Workload, kb: np.ndarray, T: np.ndarray):
    """Drafts [B, K] and uniforms [B, K+1] of a mixed batch: sequence b's drafts and uniforms
    are those of a call at its own T_b (entries past K_b are filled but never read)."""
    d = np.empty((w.B, w.K), dtype=np.int32)
    u = np.empty((w.B, w.K + 1), dtype=np.float32)
    for t in np.unique(T):
        seqs = [int(b) for b in np.flatnonzero(T == t)]
        _, Q = logits(w, seqs)
        d[seqs] = drafts(w, Q, float(t), seqs)
        u[seqs] = uniforms(w, seqs, T=float(t))
    return d, u


SEED_MARKOV = 4


def markov_table(V: int, R: int, fmt: str, seed: int = SEED_MARKOV, sd: float = 0.05):
    """A synthetic Markov-head table markov_w2 of V rows of R values, stored as the GGUF
    forms the drafter card ships: fmt "f16" -> uint16 [V, R] half-float bits; fmt "q8_0" ->
    uint8 [V, R/32 * 34] rows of blocks (float16 scale d = max|x| / 127 of the block's 32
    values, then q = round(x / d) as signed bytes). Values ~ N(0, sd), a few rows 20x wider
    so that block scales vary."""
    rng = _rng(seed, V, R)
    x = rng.normal(0.0, sd, size=(V, R)).astype(np.float32)
    wide = rng.random(V) < 0.01
    x[wide] *= 20.0
    if fmt == "f16":
        return x.astype(np.float16).view(np.uint16)
    if fmt != "q8_0":
        raise ValueError(f"unknown table format {fmt!r}")
    blocks = x.reshape(V, R // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    d = (amax / 127.0).astype(np.float16)
    d32 = d.astype(np.float32)
    inv = np.divide(1.0, d32, out=np.zeros_like(d32), where=d32 != 0)
    q = np.clip(np.rint(blocks * inv[:, :, None]), -127, 127).astype(np.int8)
    out = np.empty((V, R // 32, 34), dtype=np.uint8)
    out[:, :, 0:2] = d.view(np.uint8).reshape(V, R // 32, 2)
    out[:, :, 2:] = q.view(np.uint8)
    return out.reshape(V, (R // 32) * 34)


def markov_states(B: int, R: int, seed: int = SEED_MARKOV) -> np.ndarray:
    """Rank-R states h [B, R] float32 ~ N(0, 1)."""
    return _rng(seed, 7, B, R).normal(0.0, 1.0, size=(B, R)).astype(np.float32)


def tiny_cycles(w: Workload, cycles: int, T: float = 1.0):
    """The tiny workload's repeated-cycle form: one fixed (P, Q) pair (sequence 0's logits),
    and per cycle fresh drafts and uniforms. Returned batched as B = ``cycles`` sequences
    that share the logits, which is what running the cycles one after another computes."""
    P1, Q1 = logits(w, [0])
    P = np.repeat(P1, cycles, axis=0)
    Q = np.repeat(Q1, cycles, axis=0)
    d = np.concatenate([drafts(w, Q1, T, [0], cycle=c) for c in range(cycles)], axis=0)
    u = np.concatenate([uniforms(w, [0], T, cycle=c) for c in range(cycles)], axis=0)
    return P, Q, d, u


# ------------------------------------------------------------- parallel generation

def _fill_worker(args):
    from multiprocessing import shared_memory
    name, w, seqs, seed, p_name, q_name, T_list, d_names = args
    shp = shared_memory.SharedMemory(name=p_name)
    shq = shared_memory.SharedMemory(name=q_name)
    store = np.float32 if w.dtype == "f32" else np.uint16
    P = np.ndarray((w.B, w.K + 1, w.V), dtype=store, buffer=shp.buf)
    Q = np.ndarray((w.B, w.K, w.V), dtype=store, buffer=shq.buf)
    dsh = [shared_memory.SharedMemory(name=n) for n in d_names]
    D = [np.ndarray((w.B, w.K), dtype=np.int32, buffer=s.buf) for s in dsh]
    for b in seqs:
        p, q = logits(w, [b], seed)
        P[b], Q[b] = p[0], q[0]
        for T, d in zip(T_list, D):
            d[b] = drafts(w, q, T, [b])[0]
    del P, Q, D
    shp.close()
    shq.close()
    for s in dsh:
        s.close()
    return len(seqs)


def generate(w: Workload, temperatures=(), processes: Optional[int] = None,
             seed: int = SEED_LOGITS):
    """Whole-batch P, Q and per-temperature drafts, built by a spawn-started process pool.

    Returns (P, Q, {T: drafts}). Identical to calling ``logits`` and ``drafts`` sequence by
    sequence; only faster for the large workloads.
    """
    import multiprocessing as mp
    from multiprocessing import shared_memory

    procs = processes or min(w.B, max(1, (os.cpu_count() or 1)))
    if procs <= 1 or w.B <= 2:
        P, Q = logits(w, seed=seed)
        return P, Q, {T: drafts(w, Q, T) for T in temperatures}
    store = np.float32 if w.dtype == "f32" else np.uint16
    isz = np.dtype(store).itemsize
    shp = shared_memory.SharedMemory(create=True, size=w.B * (w.K + 1) * w.V * isz)
    shq = shared_memory.SharedMemory(create=True, size=max(1, w.B * w.K * w.V * isz))
    dsh = [shared_memory.SharedMemory(create=True, size=max(4, w.B * w.K * 4))
           for _ in temperatures]
    try:
        groups = [list(range(k, w.B, procs)) for k in range(procs)]
        args = [(w.name, w, g, seed, shp.name, shq.name, tuple(temperatures),
                 [s.name for s in dsh]) for g in groups if g]
        with mp.get_context("spawn").Pool(len(args)) as pool:
            pool.map(_fill_worker, args)
        P = np.ndarray((w.B, w.K + 1, w.V), dtype=store, buffer=shp.buf).copy()
        Q = np.ndarray((w.B, w.K, w.V), dtype=store, buffer=shq.buf).copy()
        D = {T: np.ndarray((w.B, w.K), dtype=np.int32, buffer=s.buf).copy()
             for T, s in zip(temperatures, dsh)}
    finally:
        for s in [shp, shq] + dsh:
            s.close()
            s.unlink()
    return P, Q, D
