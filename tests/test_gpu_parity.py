"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on the GPU.

Greedy: bit-exact. Sampling: probabilities within 1e-5 relative, decisions and tokens
identical except where a uniform lies within 1e-6 of a boundary (counted). Every workload
of the verify path is covered at its full size; the largest one is checked against the
oracle on sampled sequences and against properties that hold at any size.
"""

import dataclasses

import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import accept_ref as ora
from oracle import parallel as par

from gpu_helpers import (DEV, compare_greedy, compare_sampling, run_gpu, run_oracle, to_dev)

pytestmark = pytest.mark.gpu


def _small(name, **kw):
    w = wl.WORKLOADS[name]
    a = dict(B=w.B, K=w.K, V=w.V, dtype=w.dtype, kind=w.kind, params=w.params)
    a.update(kw)
    return wl.Workload(w.name, **a)


def _check(w, T, P=None, Q=None, d=None, u=None, label=""):
    if P is None:
        P, Q = wl.logits(w)
    if d is None:
        d = wl.drafts(w, Q, T)
    if u is None:
        u = wl.uniforms(w, T=T)
    g = run_gpu(P, Q, d, u, T, w.dtype)
    o = run_oracle(P, Q, d, u, T, w.dtype)
    if T == 0:
        compare_greedy(g, o)
        return 0
    return compare_sampling(g, o, label or f"{w.name} T={T}", (P, Q, u, T, w.dtype))


# ------------------------------------------------------------------ the five workloads

@pytest.mark.parametrize("T", [1.0, 0.0])
def test_tiny_1000_cycles(T):
    w = wl.WORKLOADS["tiny"]
    P, Q, d, u = wl.tiny_cycles(w, 1000, T=T)
    tw = _small("tiny", B=1000)
    near = _check(tw, T, P, Q, d, u)
    assert near <= 10


class _Same:
    """Index b of any sequence gives the one logit block that every cycle shares."""

    def __init__(self, block):
        self.block = block

    def __getitem__(self, b):
        return self.block


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_qwen3_block7(T):
    """The Qwen3-4B-shaped block at its full cycle count: 10k seeded cycles of one fixed
    logit block (fresh drafts and uniforms per cycle), verified on the GPU in batches of
    1000 cycles and by the oracle cycle by cycle."""
    w = wl.WORKLOADS["qwen3_4b_block7"]
    assert w.cycles == 10000
    _check(w, T)
    P1, Q1 = wl.logits(w)
    res = par.run(w.name, T, cycles=range(w.cycles))
    d, u = res["drafts"], res["uniforms"]
    Pd = to_dev(P1, w.dtype)
    Qd = to_dev(Q1, w.dtype)
    g = {}
    for c0 in range(0, w.cycles, 1000):
        nb = min(1000, w.cycles - c0)
        Pb = Pd.expand(nb, w.K + 1, w.V).contiguous()
        Qb = Qd.expand(nb, w.K, w.V).contiguous()
        part = run_gpu(None, None, d[c0:c0 + nb], u[c0:c0 + nb], T, w.dtype, block=Pb, Q_dev=Qb)
        for k, v in part.items():
            g.setdefault(k, []).append(v)
        del Pb, Qb
    g = {k: np.concatenate(v) for k, v in g.items()}
    o = par.as_result(res, T)
    if T == 0:
        compare_greedy(g, o)
    else:
        near = compare_sampling(g, o, f"{w.name} T={T} {w.cycles} cycles",
                                (_Same(P1[0]), _Same(Q1[0]), u, T, w.dtype))
        assert near <= 10


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_gemma4_block7(T):
    _check(wl.WORKLOADS["gemma4_12b_block7"], T)


@pytest.fixture(scope="module")
def dsv4():
    w = wl.WORKLOADS["dsv4_flash_serving"]
    P, Q, D = wl.generate(w, w.temperatures)
    return w, P, Q, D


@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
def test_dsv4_flash_serving(dsv4, T):
    w, P, Q, D = dsv4
    near = _check(w, T, P, Q, D[T], wl.uniforms(w, T=T))
    assert near <= w.B // 4


@pytest.fixture(scope="module")
def stress():
    w = wl.WORKLOADS["stress"]
    P, Q, D = wl.generate(w, w.temperatures)
    return w, P, Q, D


_STRESS_ORACLE = {}


def stress_oracle(w, T, d, u):
    """The oracle on every sequence of the stress workload at T (all host cores, once per T),
    checked to have seen the same drafts and uniforms as the GPU."""
    if T not in _STRESS_ORACLE:
        res = par.run(w.name, T, seqs=range(w.B))
        assert np.array_equal(res["drafts"], d) and np.array_equal(res["uniforms"], u)
        _STRESS_ORACLE[T] = par.as_result(res, T)
    return _STRESS_ORACLE[T]


@pytest.mark.parametrize("T", [0.0, 0.6, 1.0])
def test_stress_full_size(stress, T):
    """B256 K15 V262144 in one call, every sequence against the oracle."""
    w, P, Q, D = stress
    d, u = D[T], wl.uniforms(w, T=T)
    g = run_gpu(P, Q, d, u, T, w.dtype)
    o = stress_oracle(w, T, d, u)
    if T == 0:
        compare_greedy(g, o)
    else:
        near = compare_sampling(g, o, f"stress T={T}", (P, Q, u, T, w.dtype))
        assert near <= w.B // 4
    # every sequence: well-formed result
    n, tok = g["n_accepted"], g["tokens"]
    assert np.all(g["status"] == 0)
    assert np.all((n >= 0) & (n <= w.K))
    for b in range(w.B):
        assert np.array_equal(tok[b, : n[b]], d[b, : n[b]])
        assert 0 <= tok[b, n[b]] < w.V and tok[b, n[b]] == g["next_token"][b]
        assert np.all(tok[b, n[b] + 1:] == -1)
    if T == 0:
        # greedy at full size against the library argmax (first maximal index)
        Pd = to_dev(P, w.dtype)
        am = torch.argmax(Pd.float(), dim=-1).cpu().numpy()
        for b in range(w.B):
            j = int(n[b])
            assert np.all(d[b, :j] == am[b, :j]) and tok[b, j] == am[b, j]
            assert j == w.K or d[b, j] != am[b, j]


def _early_exit(P, Q, d, u, T, dtype):
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    r = bd.early_exit_accept(to_dev(P, dtype), to_dev(Q, dtype) if T > 0 else None, dd, T,
                             ud if T > 0 else None)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in vars(r).items() if v is not None}


def _ee_same_as_full(e, f, T, K):
    for key in ("n_accepted", "tokens", "next_token", "status"):
        assert np.array_equal(e[key], f[key]), key
    if T > 0:
        assert np.array_equal(e["resid_mass"], f["resid_mass"])
        for b in range(e["n_accepted"].shape[0]):
            t = min(int(f["n_accepted"][b]) + 1, K)
            assert np.array_equal(e["p_draft"][b, :t], f["p_draft"][b, :t])
            assert np.all(np.isnan(e["p_draft"][b, t:]))


@pytest.mark.parametrize("T", [0.0, 0.7, 1.0])
def test_dsv4_flash_serving_early_exit(dsv4, T):
    """Early exit on the serving workload: identical to the full call, and to the oracle."""
    w, P, Q, D = dsv4
    d, u = D[T], wl.uniforms(w, T=T)
    e = _early_exit(P, Q, d, u, T, w.dtype)
    _ee_same_as_full(e, run_gpu(P, Q, d, u, T, w.dtype), T, w.K)
    Pf = wl.as_float64(P, w.dtype)
    o = ora.early_exit_accept(Pf, wl.as_float64(Q, w.dtype) if T else None, d, T,
                              u.astype(np.float64) if T else None)
    if T == 0:
        compare_greedy(e, o)
    else:
        assert compare_sampling(e, o, f"ee dsv4 T={T}", (P, Q, u, T, w.dtype)) <= w.B // 4


@pytest.mark.parametrize("T", [0.0, 0.6, 1.0])
def test_stress_full_size_early_exit(stress, T):
    """B256 K15 V262144 with early exit: identical to the full call and to the oracle on every
    sequence."""
    w, P, Q, D = stress
    d, u = D[T], wl.uniforms(w, T=T)
    e = _early_exit(P, Q, d, u, T, w.dtype)
    _ee_same_as_full(e, run_gpu(P, Q, d, u, T, w.dtype), T, w.K)
    # every row of these blocks is usable, so the early-exit oracle equals the full one there
    # (pinned in test_oracle_early_exit.py): compare every sequence with it
    o = stress_oracle(w, T, d, u)
    if T == 0:
        compare_greedy(e, o)
    else:
        # p_draft / q_draft past each stop are NaN by contract (checked against the full call
        # above); compare the entries up to it
        ok = np.isfinite(e["p_draft"])
        o = dataclasses.replace(o, p_draft=np.where(ok, o.p_draft, np.nan),
                                q_draft=np.where(ok, o.q_draft, np.nan))
        compare_sampling(e, o, f"ee stress T={T}", (P, Q, u, T, w.dtype))


# --------------------------------------------------------------------- conventions

def test_block_convention_separate_buffers():
    """p_1 from the anchor step and p_2..p_{K+1} from the verify forward in two separate
    allocations (p1 with a padded row stride) give the same result as one contiguous block."""
    w = _small("dsv4_flash_serving", B=6, V=20000)
    P, Q = wl.logits(w)
    for T in (0.0, 1.0):
        d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
        whole = run_gpu(P, Q, d, u, T, w.dtype)
        Pd = to_dev(P, w.dtype)
        p1 = torch.zeros(w.B, w.V + 64, dtype=torch.bfloat16, device=DEV)[:, : w.V]
        p1.copy_(Pd[:, 0])
        pv = Pd[:, 1:].contiguous()
        split = run_gpu(None, Q, d, u, T, w.dtype, block=(p1, pv))
        for k in whole:
            assert np.array_equal(whole[k], split[k]), k


def test_q_equals_p_accepts_all_on_gpu():
    w = _small("dsv4_flash_serving", B=32, V=129280)
    P, _ = wl.logits(w)
    Q = P[:, : w.K].copy()
    for T in (0.7, 1.0, 1.3):
        d = wl.drafts(w, Q, T)
        u = wl.uniforms(w, T=T)
        g = run_gpu(P, Q, d, u, T, w.dtype)
        assert np.all(g["n_accepted"] == w.K)
        np.testing.assert_array_equal(g["p_draft"], g["q_draft"])


def test_temperature_scaling_is_exact_on_gpu():
    """(z, T) and (2z, 2T) are the same distribution; with power-of-two scaling the fp32
    arithmetic is the same too, so results are bitwise equal."""
    w = _small("dsv4_flash_serving", B=16, V=40000)
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, 0.7), wl.uniforms(w, T=0.7)
    a = run_gpu(P, Q, d, u, 0.7, w.dtype)
    P2 = wl.round_to_bf16_bits(2 * wl.as_float64(P, "bf16").astype(np.float32))
    Q2 = wl.round_to_bf16_bits(2 * wl.as_float64(Q, "bf16").astype(np.float32))
    b = run_gpu(P2, Q2, d, u, 1.4, w.dtype)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_repeated_calls_are_deterministic():
    w = _small("gemma4_12b_block7", B=4)
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, 1.0), wl.uniforms(w)
    a = run_gpu(P, Q, d, u, 1.0, w.dtype)
    b = run_gpu(P, Q, d, u, 1.0, w.dtype)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


# ---------------------------------------------------------- shapes, paths, edge cases

@pytest.mark.parametrize("V", [1, 2, 31, 1024, 1025, 4097, 50257, 130000])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_vocab_sizes(V, dtype):
    """Vocab sizes that are not multiples of the chunk; odd V forces the scalar path."""
    w = wl.Workload("r", B=5, K=4, V=V, dtype=dtype, kind="shared_noise",
                    params={"sd": 3.0, "noise": 1.0})
    for T in (0.0, 1.0):
        _check(w, T, label=f"V={V} {dtype} T={T}")


@pytest.mark.parametrize("K", [0, 1, 2, 15, 32])
def test_draft_counts(K):
    w = wl.Workload("k", B=7, K=K, V=3000, dtype="bf16", kind="shared_noise",
                    params={"sd": 2.0, "noise": 0.5})
    for T in (0.0, 0.8):
        _check(w, T, label=f"K={K} T={T}")


def test_many_sequences_small_vocab():
    w = wl.Workload("m", B=3000, K=3, V=64, dtype="f32", kind="iid", params={"sd": 2.0})
    for T in (0.0, 1.0):
        _check(w, T)


def test_empty_batch_is_a_noop():
    P = torch.zeros(0, 4, 128, dtype=torch.bfloat16, device=DEV)
    d = torch.zeros(0, 3, dtype=torch.int32, device=DEV)
    u = torch.zeros(0, 4, dtype=torch.float32, device=DEV)
    assert bd.greedy_accept(P, d).n_accepted.numel() == 0
    Q = torch.zeros(0, 3, 128, dtype=torch.bfloat16, device=DEV)
    assert bd.speculative_sample_accept(P, Q, d, 1.0, u).n_accepted.numel() == 0


def test_data_errors_reported_per_sequence():
    w = wl.Workload("e", B=8, K=3, V=5000, dtype="f32", kind="shared_noise",
                    params={"sd": 2.0, "noise": 1.0})
    P, Q = wl.logits(w)
    P, Q = P.copy(), Q.copy()
    d = wl.drafts(w, Q, 1.0)
    u = wl.uniforms(w)
    d[0, 1] = w.V              # draft id out of range
    d[1, 2] = -3
    P[2, 3, 17] = np.nan       # NaN in the bonus row
    Q[3, 0, :] = -np.inf       # a draft row with no finite value
    P[4, 1, 100] = np.inf      # +inf
    P[5, 0, :4000] = -np.inf   # masked tokens are fine
    P[6, 2, :] = -np.inf       # a base row with no finite value
    for T in (0.0, 1.0):
        g = run_gpu(P, Q, d, u, T, w.dtype)
        o = run_oracle(P, Q, d, u, T, w.dtype)
        if T == 0:
            compare_greedy(g, o)
        else:
            compare_sampling(g, o, "errors", (P, Q, u, T, w.dtype))
        assert (g["status"][5] & (bd.SEQ_BAD_DRAFT | bd.SEQ_NONFINITE)) == 0
        assert np.all(g["tokens"][[0, 1, 2, 4, 6]] == -1)


def test_chi_square_first_token_one_million_cycles():
    """Tiny workload, 10^6 GPU cycles (drafts drawn from q with torch.multinomial): the first
    emitted token follows p_1, and the mean accepted count matches sum_k prod_{i<k} alpha_i."""
    from scipy import special, stats
    w = wl.WORKLOADS["tiny"]
    P1, Q1 = wl.logits(w)
    N = 1_000_000
    gen = torch.Generator(device=DEV)
    gen.manual_seed(1234)
    Pd = to_dev(P1, "f32").expand(N, -1, -1).contiguous()
    Qd = to_dev(Q1, "f32").expand(N, -1, -1).contiguous()
    q = torch.softmax(Qd[0].double(), dim=-1)
    d = torch.stack([torch.multinomial(q[i], N, replacement=True, generator=gen)
                     for i in range(w.K)], dim=1).to(torch.int32).contiguous()
    u = torch.rand(N, w.K + 1, generator=gen, device=DEV, dtype=torch.float32)
    r = bd.speculative_sample_accept(Pd, Qd, d, 1.0, u)
    first = r.tokens[:, 0].long().cpu().numpy()
    p = special.softmax(P1[0].astype(np.float64), axis=-1)
    qq = special.softmax(Q1[0].astype(np.float64), axis=-1)
    obs = np.bincount(first, minlength=w.V)
    exp = p[0] * N
    keep = exp >= 5
    o2, e2 = obs[keep], exp[keep]
    if (~keep).any():
        o2 = np.append(o2, obs[~keep].sum())
        e2 = np.append(e2, exp[~keep].sum())
    e2 = e2 * (o2.sum() / e2.sum())
    assert stats.chisquare(o2, e2).pvalue > 1e-3
    alpha = [np.minimum(p[i], qq[i]).sum() for i in range(w.K)]
    expect = sum(np.prod(alpha[:k]) for k in range(1, w.K + 1))
    n = r.n_accepted.double()
    assert abs(n.mean().item() - expect) < 4 * n.std().item() / np.sqrt(N)


def test_shared_workspace_across_growing_batches():
    """The binding's shared workspace: a small batch, then a larger one whose per-sequence
    counters lie where the small call kept its records; results must not depend on it."""
    small = wl.Workload("s", B=5, K=3, V=4096, dtype="bf16", kind="shared_noise",
                        params={"sd": 2.0, "noise": 1.0})
    big = wl.Workload("g", B=700, K=3, V=64, dtype="f32", kind="iid", params={"sd": 2.0})
    for w in (small, big, small, big):
        _check(w, 1.0, label=f"{w.name} B={w.B}")
