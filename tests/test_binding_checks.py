"""The Python binding's layout checks, without a GPU.

The C library checks its pointers for null but cannot see the sizes behind them, so every
wrapper checks shapes, dtypes, contiguity and devices first: a short ``uniforms`` or result
tensor must raise ValueError before any pointer reaches the library. These calls use CPU
tensors, so a call that passes every layout check ends in the wrappers' CUDA-only error.
"""

import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import build_lib

B, K, V = 2, 3, 64


@pytest.fixture(scope="module", autouse=True)
def lib():
    build_lib.build()
    return bd.load_library()


def _args(**over):
    a = dict(P=torch.zeros(B, K + 1, V, dtype=torch.bfloat16),
             Q=torch.zeros(B, K, V, dtype=torch.bfloat16),
             drafts=torch.zeros(B, K, dtype=torch.int32),
             uniforms=torch.zeros(B, K + 1, dtype=torch.float32))
    a.update(over)
    return a


def _out(**over):
    i32, f32 = dict(dtype=torch.int32), dict(dtype=torch.float32)
    o = dict(n_accepted=torch.zeros(B, **i32), tokens=torch.zeros(B, K + 1, **i32),
             next_token=torch.zeros(B, **i32), status=torch.zeros(B, **i32),
             p_draft=torch.zeros(B, K, **f32), q_draft=torch.zeros(B, K, **f32),
             resid_mass=torch.zeros(B, **f32))
    o.update(over)
    return bd.AcceptResult(**o)


def _static(out=None, T=1.0, **over):
    a = _args(**over)
    return bd.speculative_sample_accept_static(a["P"], a["Q"], a["drafts"], T, a["uniforms"],
                                               out=out if out is not None else _out())


def test_static_wrapper_accepts_well_formed_arguments_up_to_the_cuda_check():
    with pytest.raises(RuntimeError, match="CUDA tensors only"):
        _static()


@pytest.mark.parametrize("bad", [
    dict(uniforms=torch.zeros(B, K, dtype=torch.float32)),          # one uniform short
    dict(uniforms=torch.zeros(B - 1, K + 1, dtype=torch.float32)),  # one sequence short
    dict(uniforms=torch.zeros(B, K + 1, dtype=torch.float64)),      # wrong dtype
    dict(uniforms=torch.zeros(K + 1, B, dtype=torch.float32).t()),  # not contiguous
    dict(Q=None),
    dict(Q=torch.zeros(B, K - 1, V, dtype=torch.bfloat16)),
    dict(Q=torch.zeros(B, K, V, dtype=torch.float32)),
    dict(drafts=torch.zeros(B, K - 1, dtype=torch.int32)),
])
def test_static_wrapper_rejects_bad_inputs(bad):
    with pytest.raises(ValueError):
        _static(**bad)


@pytest.mark.parametrize("field,t", [
    ("n_accepted", torch.zeros(B - 1, dtype=torch.int32)),
    ("tokens", torch.zeros(B, K, dtype=torch.int32)),             # one token short
    ("tokens", torch.zeros(B, K + 1, dtype=torch.int64)),
    ("next_token", None),
    ("status", torch.zeros(B + 1, dtype=torch.int32)),
    ("p_draft", torch.zeros(B, K - 1, dtype=torch.float32)),
    ("q_draft", torch.zeros(B, K, dtype=torch.float16)),
    ("resid_mass", torch.zeros(2 * B, dtype=torch.float32)[::2]),  # not contiguous
])
def test_static_wrapper_rejects_bad_results(field, t):
    with pytest.raises(ValueError):
        _static(out=_out(**{field: t}))


def test_static_wrapper_requires_out():
    a = _args()
    with pytest.raises(ValueError, match="out is required"):
        bd.speculative_sample_accept_static(a["P"], a["Q"], a["drafts"], 1.0, a["uniforms"],
                                            out=None)


def test_optional_result_fields_may_be_absent():
    with pytest.raises(RuntimeError, match="CUDA tensors only"):
        _static(out=_out(status=None, p_draft=None, q_draft=None, resid_mass=None))


def test_greedy_at_zero_temperature_needs_no_uniforms():
    with pytest.raises(RuntimeError, match="CUDA tensors only"):
        _static(T=0.0, uniforms=None, Q=None)


def test_markov_wrappers_check_before_launch():
    """markov_matvec and its test-only withheld variant reject an unknown table format and a
    table that is not on the GPU before anything reaches the library."""
    table = torch.zeros(16, 272, dtype=torch.uint8)
    h = torch.zeros(1, 256, dtype=torch.float32)
    for fn in (bd.markov_matvec, bd.markov_matvec_withheld):
        with pytest.raises(ValueError, match="fmt"):
            fn(table, "q4_0", h)
        with pytest.raises(ValueError, match="CUDA"):
            fn(table, "q8_0", h)
