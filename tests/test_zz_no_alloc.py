"""The entry point without a workspace (fixed per-device scratch in the library's image).

It must give what the workspace entry point gives on the same inputs, on consecutive calls,
whether it runs first in a fresh process (its first call looks up the scratch address) or
after every other test. Shapes beyond the fixed scratch are rejected before any CUDA work.
"""


import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import build_lib
from lossless_draft_verification_speculative_b200 import workloads as wl

BF16 = 0
FAKE = 0x10000  # a fake device address: the rejected calls below never dereference it
PROB_RTOL = 1e-5


def _lib():
    build_lib.build()
    return bd.load_library()


def _static_call(lib, B, K, V, T=1.0):
    out = bd.AcceptOut(FAKE, FAKE, FAKE, None, None, None, None)
    return lib.dspark_speculative_sample_accept_static(
        FAKE, V, FAKE, K * V, FAKE, BF16, FAKE, B, K, V, T, FAKE, out, None)


def test_oversized_shape_is_rejected_before_any_cuda_work():
    lib = _lib()
    assert bd.STATIC_SCRATCH_BYTES == 4 << 20
    big = (256, 15, 262144)
    assert lib.dspark_workspace_bytes(*big, BF16) > bd.STATIC_SCRATCH_BYTES
    assert _static_call(lib, *big) == 4                       # DSPARK_ERR_WORKSPACE
    assert _static_call(lib, *big, T=0.0) == 4
    assert lib.dspark_workspace_bytes(64, 7, 129280, BF16) <= bd.STATIC_SCRATCH_BYTES
    assert _static_call(lib, 64, 7, 129280, T=-1.0) == 1      # argument checks still apply
    assert _static_call(lib, 0, 7, 129280) == 0               # empty batch: a no-op


def _inputs(B, K, V, seed):
    w = wl.Workload("no_alloc", B=B, K=K, V=V, dtype="bf16", kind="shared_noise",
                    params={"sd": 2.0, "noise": 0.7})
    P, Q = wl.logits(w, seed=seed)
    d = wl.drafts(w, Q, 1.0, seed=seed + 1)
    u = wl.uniforms(w, seed=seed + 2)
    dev = "cuda:0"
    Pd = torch.from_numpy(np.ascontiguousarray(P).view(np.int16)).to(dev).view(torch.bfloat16)
    Qd = torch.from_numpy(np.ascontiguousarray(Q).view(np.int16)).to(dev).view(torch.bfloat16)
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(dev)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(dev)
    return Pd, Qd, dd, ud


def _result(B, K):
    dev = "cuda:0"
    i32 = dict(dtype=torch.int32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    return bd.AcceptResult(n_accepted=torch.full((B,), -7, **i32),
                           tokens=torch.full((B, K + 1), -7, **i32),
                           next_token=torch.full((B,), -7, **i32),
                           status=torch.full((B,), -7, **i32),
                           p_draft=torch.full((B, K), -7.0, **f32),
                           q_draft=torch.full((B, K), -7.0, **f32),
                           resid_mass=torch.full((B,), -7.0, **f32))


def _static(lib, P, Q, d, u, T, out):
    p1, pv, ld_p1, ld_pv = bd._split_block(P)
    B, V = p1.shape
    K = pv.shape[1]
    rc = lib.dspark_speculative_sample_accept_static(
        p1.data_ptr(), ld_p1, pv.data_ptr(), ld_pv, Q.data_ptr(), BF16, d.data_ptr(), B, K, V,
        T, u.data_ptr(), bd._out_struct(out), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, bd.STATUS_NAMES.get(rc, rc)
    return out


def _same(a, b, T):
    for k in ("n_accepted", "tokens", "next_token", "status"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k
    if T > 0:
        for k in ("p_draft", "q_draft", "resid_mass"):
            x, y = getattr(a, k).double().cpu(), getattr(b, k).double().cpu()
            np.testing.assert_allclose(x.numpy(), y.numpy(), rtol=PROB_RTOL, atol=1e-37,
                                       err_msg=k)


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1.0, 0.0])
def test_static_scratch_matches_workspace_entry_on_consecutive_calls(T):
    lib = _lib()
    # two calls in a row, different shapes, so the second one starts from the first one's
    # leftovers in the scratch
    cases = [(64, 7, 129280, 11), (9, 3, 50000, 23)]
    for B, K, V, seed in cases:
        P, Q, d, u = _inputs(B, K, V, seed)
        mine = _static(lib, P, Q, d, u, T, _result(B, K))
        if T == 0:
            ref = bd.greedy_accept(P, d, out=_result(B, K))
        else:
            ref = bd.speculative_sample_accept(P, Q, d, T, u, out=_result(B, K))
        torch.cuda.synchronize()
        assert int((mine.n_accepted < 0).sum()) == 0
        _same(mine, ref, T)
