"""The early-exit verify step on the GPU.

Against the oracle's ``early_exit_accept`` (greedy bit-exact, sampling within the tolerances of
the single-policy tests) and against the full call on the same inputs: the waves write the
records of a full call and decide with its arithmetic, so on blocks whose rows are all usable
every output up to the stop is bit-identical. Rows after a sequence's stop are never read:
poisoning them changes nothing.
"""


import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl
from oracle import accept_ref as ora

from gpu_helpers import DEV, compare_greedy, compare_sampling, run_gpu, to_dev

pytestmark = pytest.mark.gpu


def run_ee(P, Q, d, u, T, dtype):
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    Qd = to_dev(Q, dtype) if (T > 0 and d.shape[1] > 0) else None
    r = bd.early_exit_accept(to_dev(P, dtype), Qd, dd, T, ud if T > 0 else None)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in vars(r).items() if v is not None}


def oracle_ee(P, Q, d, u, T, dtype):
    Qf = wl.as_float64(Q, dtype) if T > 0 else None
    return ora.early_exit_accept(wl.as_float64(P, dtype), Qf, d, T,
                                 u.astype(np.float64) if T > 0 else None)


def same_as_full(e, f, T):
    """Bit-identical to the full call: every result, and p_draft / q_draft up to the stop."""
    for key in ("n_accepted", "tokens", "next_token", "status"):
        assert np.array_equal(e[key], f[key]), key
    if T > 0:
        K = e["p_draft"].shape[1]
        assert np.array_equal(e["resid_mass"], f["resid_mass"], equal_nan=True)
        for b in range(e["n_accepted"].shape[0]):
            if f["status"][b] & (bd.SEQ_BAD_DRAFT | bd.SEQ_NONFINITE):
                continue
            t = min(int(f["n_accepted"][b]) + 1, K)
            for key in ("p_draft", "q_draft"):
                assert np.array_equal(e[key][b, :t], f[key][b, :t]), (key, b)
                assert np.all(np.isnan(e[key][b, t:])), (key, b)


def _workload(B, K, V, dtype, sigmas=(0.25, 1.0, 4.0)):
    return wl.Workload("ee", B=B, K=K, V=V, dtype=dtype, kind="mixed_sigma",
                       params={"sd": 3.0, "sigmas": sigmas})


@pytest.mark.parametrize("K", [0, 1, 2, 3, 7, 15, 32])
@pytest.mark.parametrize("T", [0.0, 1.0])
def test_draft_counts_against_oracle_and_full_call(K, T):
    w = _workload(24, K, 3000, "bf16")
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
    e = run_ee(P, Q, d, u, T, w.dtype)
    o = oracle_ee(P, Q, d, u, T, w.dtype)
    if T == 0:
        compare_greedy(e, o)
    else:
        compare_sampling(e, o, f"ee K={K}", (P, Q, u, T, w.dtype))
    same_as_full(e, run_gpu(P, Q, d, u, T, w.dtype), T)


@pytest.mark.parametrize("V,dtype", [(1, "f32"), (2047, "bf16"), (2049, "f32"), (5001, "bf16"),
                                     (65536, "bf16")])
@pytest.mark.parametrize("T", [0.0, 0.7])
def test_ragged_vocab_sizes(V, dtype, T):
    w = _workload(9, 5, V, dtype)
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
    e = run_ee(P, Q, d, u, T, dtype)
    o = oracle_ee(P, Q, d, u, T, dtype)
    if T == 0:
        compare_greedy(e, o)
    else:
        compare_sampling(e, o, f"ee V={V}", (P, Q, u, T, dtype))
    same_as_full(e, run_gpu(P, Q, d, u, T, dtype), T)


@pytest.mark.parametrize("ctas", ["1", "3", "37"])
def test_pass_one_grid_sizes(ctas, monkeypatch):
    """The wave's unit walk and its look-ahead of the next unit's sequence with few CTAs."""
    w = _workload(40, 7, 9000, "bf16")
    P, Q = wl.logits(w)
    for T in (0.0, 1.0):
        d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
        full = run_gpu(P, Q, d, u, T, w.dtype)
        monkeypatch.setenv("DSPARK_MAX_CTAS", ctas)
        e = run_ee(P, Q, d, u, T, w.dtype)
        monkeypatch.delenv("DSPARK_MAX_CTAS")
        same_as_full(e, full, T)


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_rows_after_the_stop_are_not_read(T):
    w = _workload(48, 7, 4096, "bf16")
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
    clean = run_ee(P, Q, d, u, T, w.dtype)
    nan = np.uint16(0x7fc0)
    P2, Q2 = P.copy(), Q.copy()
    cut = 0
    for b in range(w.B):
        j = int(clean["n_accepted"][b])
        if j < w.K:
            P2[b, j + 1:] = nan
            Q2[b, j + 1:] = nan
            cut += 1
    assert cut >= 10
    e = run_ee(P2, Q2, d, u, T, w.dtype)
    for key in ("n_accepted", "tokens", "next_token", "status"):
        assert np.array_equal(e[key], clean[key]), key
    full = run_gpu(P2, Q2, d, u, T, w.dtype)  # the full call reads them and reports them
    assert np.sum(full["status"] & bd.SEQ_NONFINITE != 0) == cut


@pytest.mark.parametrize("T", [0.0, 1.0])
def test_errors(T):
    """A bad row at or before the stop, a bad bonus row after a full accept, a bad draft id."""
    w = _workload(6, 3, 2048, "f32", sigmas=(0.25,))
    P, Q = wl.logits(w)
    d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
    am = wl.as_float64(P, "f32").argmax(axis=2)
    d[:] = am[:, :3]               # greedy accepts every draft
    u[:, :3] = 0.0                 # sampling accepts every draft with q > 0
    P[1, 0, 5] = np.nan            # row 0 is read and is before the stop
    P[2, 3, :] = -np.inf           # the bonus row, read after a full accept
    d[3, 2] = w.V                  # a bad id: nothing read
    P[3] = np.nan
    P[4, 1, 7] = np.inf            # +inf in row 1
    e = run_ee(P, Q, d, u, T, "f32")
    o = oracle_ee(P, Q, d, u, T, "f32")
    assert list(o.status) == [0, 2, 2, 1, 2, 0]
    assert np.array_equal(e["status"] & 3, o.status)
    for b in (1, 2, 3, 4):
        assert e["n_accepted"][b] == 0 and e["next_token"][b] == -1 and np.all(e["tokens"][b] == -1)
    for b in (0, 5):
        assert e["n_accepted"][b] == 3 and np.array_equal(e["tokens"][b, :3], d[b])


def test_empty_batch_is_a_noop():
    P = torch.empty(0, 4, 64, device=DEV)
    d = torch.empty(0, 3, dtype=torch.int32, device=DEV)
    r = bd.early_exit_accept(P, torch.empty(0, 3, 64, device=DEV), d, 1.0,
                             torch.empty(0, 4, device=DEV))
    assert r.n_accepted.numel() == 0


def test_shared_workspace_between_policies():
    """One workspace serves early-exit and full calls back to back, in any order."""
    w = _workload(32, 7, 8192, "bf16")
    P, Q = wl.logits(w)
    Pd, Qd = to_dev(P, "bf16"), to_dev(Q, "bf16")
    ws = bd.new_workspace(bd.workspace_bytes(w.B, w.K, w.V, torch.bfloat16), DEV)
    for T in (1.0, 0.0, 0.7):
        dd = torch.from_numpy(wl.drafts(w, Q, T)).to(DEV)
        ud = torch.from_numpy(wl.uniforms(w, T=T)).to(DEV)
        a = bd.early_exit_accept(Pd, Qd, dd, T, ud, workspace=ws)
        f = bd.speculative_sample_accept(Pd, Qd, dd, T, ud, workspace=ws)
        b = bd.early_exit_accept(Pd, Qd, dd, T, ud, workspace=ws)
        torch.cuda.synchronize()
        for x, y in ((a, f), (a, b)):
            assert torch.equal(x.n_accepted, y.n_accepted) and torch.equal(x.tokens, y.tokens)
