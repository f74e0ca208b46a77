"""The seeded input generators: rounding, determinism, shapes, draft law."""

import numpy as np
import torch
from scipy import special, stats

from lossless_draft_verification_speculative_b200 import workloads as wl


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 30, 100000), rng.normal(0, 1e-3, 1000),
                        [0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38]]).astype(np.float32)
    ours = wl.round_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = wl.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_per_sequence_generation_is_independent_of_the_batch():
    w = wl.WORKLOADS["dsv4_flash_serving"]
    small = wl.Workload(w.name, B=6, K=2, V=300, dtype=w.dtype, kind=w.kind, params=w.params)
    P_all, Q_all = wl.logits(small)
    P_sub, Q_sub = wl.logits(small, [4, 1])
    assert np.array_equal(P_all[[4, 1]], P_sub) and np.array_equal(Q_all[[4, 1]], Q_sub)
    d_all = wl.drafts(small, Q_all, 0.7)
    d_sub = wl.drafts(small, Q_sub, 0.7, seqs=[4, 1])
    assert np.array_equal(d_all[[4, 1]], d_sub)
    u_all = wl.uniforms(small, T=0.7)
    assert np.array_equal(u_all[[4, 1]], wl.uniforms(small, [4, 1], T=0.7))
    assert u_all.dtype == np.float32 and np.all((u_all >= 0) & (u_all < 1))


def test_every_recipe_shapes_and_dtypes():
    for name, w in wl.WORKLOADS.items():
        small = wl.Workload(w.name, B=2, K=w.K, V=min(w.V, 512), dtype=w.dtype, kind=w.kind,
                            params=w.params)
        P, Q = wl.logits(small)
        assert P.shape == (2, w.K + 1, small.V) and Q.shape == (2, w.K, small.V)
        assert P.dtype == (np.float32 if w.dtype == "f32" else np.uint16)
        Pf = wl.as_float64(P, w.dtype)
        assert np.all(np.isfinite(Pf))
        if w.kind == "softcap":
            assert np.all(np.abs(Pf) <= 30.0)


def test_draft_law_is_softmax_of_q():
    """Gumbel-max drafts follow softmax(Q/T) (chi-square on a 10-token row)."""
    w = wl.Workload("t", B=1, K=1, V=10, dtype="f32", kind="iid", params={"sd": 1.0})
    _, Q = wl.logits(w)
    T = 0.8
    counts = np.zeros(w.V)
    for c in range(4000):
        counts[wl.drafts(w, Q, T, cycle=c)[0, 0]] += 1
    p = special.softmax(Q[0, 0].astype(np.float64) / T)
    assert stats.chisquare(counts, p * counts.sum()).pvalue > 1e-3


def test_greedy_drafts_are_argmax():
    w = wl.Workload("t", B=3, K=4, V=100, dtype="bf16", kind="shared_noise",
                    params={"sd": 3.0, "noise": 1.0})
    _, Q = wl.logits(w)
    d = wl.drafts(w, Q, 0.0)
    assert np.array_equal(d, np.argmax(wl.as_float64(Q, "bf16"), axis=-1))
