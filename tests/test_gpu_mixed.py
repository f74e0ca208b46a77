"""Mixed serving batches on the GPU against the oracle's ``mixed_accept``.

Each sequence verifies its own number of drafts K_b <= K at its own temperature T_b (greedy
where T_b == 0). Greedy sequences are bit-exact; sampling sequences follow the tolerances of
the single-policy tests. Rows, drafts and uniforms past a sequence's K_b are never read, so
the tests fill them with NaN, out-of-range ids and junk; a bad K_b or T_b is an error of its
own sequence only.
"""

import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import accept_ref as ora

from gpu_helpers import DEV, compare_greedy, compare_sampling, to_dev

pytestmark = pytest.mark.gpu

ERR = bd.SEQ_BAD_DRAFT | bd.SEQ_NONFINITE | bd.SEQ_BAD_PARAM


def _gpu(P, Q, d, kb, T, u, dtype):
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    Td = torch.from_numpy(np.ascontiguousarray(T, dtype=np.float32)).to(DEV)
    kd = None if kb is None else torch.from_numpy(np.ascontiguousarray(kb, dtype=np.int32)).to(DEV)
    r = bd.mixed_accept(to_dev(P, dtype), to_dev(Q, dtype), dd, Td, ud, n_drafts=kd)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in vars(r).items() if v is not None}


def _compare(g, o, P, Q, u, kb, T, dtype, label):
    """Greedy sequences bit-exact, sampling sequences within tolerance, errors identical."""
    B, K = g["tokens"].shape[0], g["tokens"].shape[1] - 1
    assert np.array_equal(g["status"] & ERR, o.status & ERR), label
    near = 0
    for b in range(B):
        if o.status[b] & ERR:
            assert g["n_accepted"][b] == 0 and g["next_token"][b] == -1, (label, b)
            assert np.all(g["tokens"][b] == -1), (label, b)
            continue
        k = K if kb is None else int(kb[b])
        sub = lambda a: {key: v[b:b + 1] for key, v in a.items()}  # noqa: E731
        ob = ora.OracleResult(o.n_accepted[b:b + 1], o.tokens[b:b + 1], o.next_token[b:b + 1],
                              o.status[b:b + 1], p_draft=o.p_draft[b:b + 1, :k],
                              q_draft=o.q_draft[b:b + 1, :k], resid_mass=o.resid_mass[b:b + 1],
                              accept_margin=o.accept_margin[b:b + 1, :k],
                              cdf_margin=o.cdf_margin[b:b + 1])
        gb = sub(g)
        if T[b] == 0:
            compare_greedy(gb, ob)
            continue
        # the single-policy comparison on the sequence's own block (tokens cut to K_b + 1)
        gb = dict(gb, tokens=gb["tokens"][:, :k + 1], p_draft=gb["p_draft"][:, :k],
                  q_draft=gb["q_draft"][:, :k])
        ob.tokens = ob.tokens[:, :k + 1]
        assert np.all(g["tokens"][b, k + 1:] == -1), (label, b)
        near += compare_sampling(gb, ob, f"{label} b={b}",
                                 (P[b:b + 1, :k + 1], Q[b:b + 1, :k], u[b:b + 1, :k + 1],
                                  float(T[b]), dtype))
    return near


def _case(name, B, K, V, dtype, kind, params, temps=(0.0, 0.7, 1.0), poison=True):
    w = wl.Workload(name, B=B, K=K, V=V, dtype=dtype, kind=kind, params=params)
    kb, T = wl.mixed_params(w, temps)
    P, Q = wl.logits(w)
    d, u = wl.mixed_inputs(w, kb, T)
    if poison:  # never read: rows, drafts and uniforms past each sequence's count
        nan = np.float32(np.nan) if dtype == "f32" else np.uint16(0x7fc0)
        for b in range(B):
            P[b, kb[b] + 1:] = nan
            Q[b, kb[b]:] = nan
            if T[b] == 0:
                Q[b] = nan
            d[b, kb[b]:] = V + 11
            u[b, kb[b] + 1:] = 2.0
    g = _gpu(P, Q, d, kb, T, u, dtype)
    o = ora.mixed_accept(wl.as_float64(P, dtype), wl.as_float64(Q, dtype), d, kb, T,
                         u.astype(np.float64))
    return _compare(g, o, P, Q, u, kb, T, dtype, name)


def test_serving_shape_mixed_batch():
    near = _case("dsv4_mixed", 64, 7, 129280, "bf16", "mixed_sigma",
                 {"sd": 3.0, "sigmas": [0.25, 1.0, 4.0]})
    assert near <= 16


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("V", [64, 4097, 50257])
def test_ragged_mixed_batches(dtype, V):
    _case(f"mixed_{V}", 40, 5, V, dtype, "shared_noise", {"sd": 2.0, "noise": 1.0})


def test_long_blocks_and_all_sampling():
    _case("mixed_k32", 12, 32, 3000, "bf16", "shared_noise", {"sd": 2.0, "noise": 0.5},
          temps=(0.6, 1.0, 1.5))


def test_all_greedy_mixed_batch():
    _case("mixed_greedy", 30, 7, 9000, "bf16", "iid", {"sd": 2.0}, temps=(0.0,))


def test_counts_default_to_k_and_match_the_single_policy_call():
    """n_drafts = NULL and one temperature: the same results as speculative_sample_accept."""
    w = wl.Workload("uni", B=16, K=7, V=20000, dtype="bf16", kind="shared_noise",
                    params={"sd": 3.0, "noise": 1.0})
    P, Q = wl.logits(w)
    d = wl.drafts(w, Q, 1.0)
    u = wl.uniforms(w, T=1.0)
    g = _gpu(P, Q, d, None, np.ones(16, dtype=np.float32), u, "bf16")
    dd = torch.from_numpy(d).to(DEV)
    r = bd.speculative_sample_accept(to_dev(P, "bf16"), to_dev(Q, "bf16"), dd, 1.0,
                                     torch.from_numpy(u).to(DEV))
    torch.cuda.synchronize()
    for k in ("n_accepted", "tokens", "next_token", "status"):
        assert np.array_equal(g[k], getattr(r, k).cpu().numpy()), k
    for k in ("p_draft", "q_draft", "resid_mass"):
        assert np.array_equal(g[k], getattr(r, k).cpu().numpy()), k


def test_bad_counts_and_temperatures_are_per_sequence_errors():
    B, K, V = 8, 3, 5000
    w = wl.Workload("bad", B=B, K=K, V=V, dtype="bf16", kind="iid", params={"sd": 2.0})
    P, Q = wl.logits(w)
    d = wl.drafts(w, Q, 1.0)
    u = wl.uniforms(w, T=1.0)
    kb = np.array([-1, K + 1, 2, 2, 2, 2, 1, 0], dtype=np.int32)
    T = np.array([1, 1, -0.5, np.nan, np.inf, 1e-45, 0.0, 0.9], dtype=np.float32)
    g = _gpu(P, Q, d, kb, T, u, "bf16")
    o = ora.mixed_accept(wl.as_float64(P, "bf16"), wl.as_float64(Q, "bf16"), d, kb,
                         T.astype(np.float64), u.astype(np.float64))
    for b in range(6):
        assert g["status"][b] == bd.SEQ_BAD_PARAM, b
        assert g["n_accepted"][b] == 0 and np.all(g["tokens"][b] == -1)
    # 1e-45 is a valid temperature for the oracle but log2(e)/T overflows float32 on the GPU
    assert o.status[5] == 0
    _compare({k: v[6:] for k, v in g.items()},
             ora.mixed_accept(wl.as_float64(P[6:], "bf16"), wl.as_float64(Q[6:], "bf16"), d[6:],
                              kb[6:], T[6:].astype(np.float64), u[6:].astype(np.float64)),
             P[6:], Q[6:], u[6:], kb[6:], T[6:], "bf16", "bad")
