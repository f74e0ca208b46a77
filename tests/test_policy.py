"""The yield-quench speculation policy (include/dspark_policy.h) on the host, no GPU.

The DeepSeek-V4-Flash DSpark drafter card (closing paragraph of "Usage") bounds the variance
of speculation with a terminal yield-quench controller, off per request when acceptance
cannot pay the verify cost (worst case about 0.96x plain decode), and a kv-depth gate that
hands requests of more than 64k tokens of context to plain decode. These tests drive the
library's controller with scripted acceptance traces and check those properties, plus the
closed form of the worst case.
"""

import ctypes

import numpy as np
import pytest

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import build_lib


@pytest.fixture(scope="module", autouse=True)
def lib():
    build_lib.build()
    return bd.load_library()


def _run(trace, break_even=1.5, warmup=8, window=16, kv=None, kv_limit=65536):
    """Feed one request's n_accepted per step; returns the speculate flags after each step."""
    q = bd.YieldQuench(1, break_even, warmup, window, kv_limit)
    flags = []
    for t, n in enumerate(trace):
        kvd = None if kv is None else np.asarray([kv[t]], dtype=np.int64)
        flags.append(bool(q.update(np.asarray([n], dtype=np.int32), kvd)[0]))
    return flags, q


def test_high_acceptance_keeps_speculating():
    # the card's mean commit of 3.70 per cycle (n_accepted 2-3 ...) against a 1.5-step cycle
    rng = np.random.default_rng(0)
    trace = rng.choice([1, 2, 3, 4, 5, 7], size=500, p=[.1, .2, .25, .2, .15, .1])
    flags, q = _run(trace)
    assert all(flags)
    assert q.state(0)["cycles"] == 500 and q.state(0)["committed"] == int((trace + 1).sum())


def test_low_acceptance_is_quenched_after_the_warmup_and_stays_off():
    trace = [0] * 8 + [7] * 50          # nothing accepted, then (too late) everything
    flags, q = _run(trace, warmup=8)
    assert flags[:7] == [True] * 7      # not judged before the warmup
    assert flags[7] is False            # judged at cycle 8: mean yield 1 < 1.5
    assert not any(flags[8:])           # terminal: the later full accepts are never seen
    assert q.state(0)["state"] == bd.SPEC_OFF_YIELD and q.state(0)["cycles"] == 8


def test_trailing_window_catches_a_drop():
    trace = [4] * 40 + [0] * 40          # commits 5 per cycle, then 1
    flags, q = _run(trace, break_even=1.5, window=16)
    # the window mean falls below 1.5 once fewer than (1.5 - 1) * 16 / 4 = 2 of the last 16
    # cycles are good ones: at the 15th bad cycle (mean (1*5 + 15*1)/16 = 1.25 < 1.5)
    first_off = flags.index(False)
    window = trace[first_off - 15:first_off + 1]
    assert np.mean(np.asarray(window) + 1) < 1.5
    prev = trace[first_off - 16:first_off]
    assert np.mean(np.asarray(prev) + 1) >= 1.5
    assert first_off == 40 + 14 and not any(flags[first_off:])


def test_exact_break_even_keeps_speculating():
    # mean yield exactly equal to the break-even: speculation is as fast as plain decode, and
    # the controller only quenches strictly below it
    flags, _ = _run([1, 0] * 50, break_even=1.5, window=2, warmup=2)
    assert all(flags)
    flags, _ = _run([1, 0] * 50, break_even=1.5 + 1e-9, window=2, warmup=2)
    assert flags.index(False) == 1


def test_unverified_steps_do_not_count():
    flags, q = _run([-1] * 30 + [0] * 7, warmup=8)
    assert all(flags) and q.state(0)["cycles"] == 7


def test_kv_depth_gate_hands_long_contexts_to_plain_decode():
    kv = [65000, 65536, 65537, 10]      # the gate is "more than 64k"; the state stays off
    flags, q = _run([7, 7, 7, 7], kv=kv)
    assert flags == [True, True, False, False]
    assert q.state(0)["state"] == bd.SPEC_OFF_KV
    flags, _ = _run([7] * 4, kv=[10 ** 9] * 4, kv_limit=0)   # 0: no gate
    assert all(flags)


def test_batch_of_requests_is_independent():
    q = bd.YieldQuench(3, 1.5, warmup=2, window=4)
    seq = [np.asarray([3, 0, -1], np.int32), np.asarray([3, 0, 0], np.int32),
           np.asarray([3, 5, 0], np.int32)]
    outs = [q.update(n, np.asarray([100, 100, 70000], np.int64)) for n in seq]
    assert outs[0].tolist() == [True, True, False]   # request 2 gated at once
    assert outs[1].tolist() == [True, False, False]  # request 1: mean yield 1 after 2 cycles
    assert outs[2].tolist() == [True, False, False]
    assert q.state(2)["cycles"] == 0                 # gated before any verified cycle


def test_worst_case_slowdown_matches_the_closed_form():
    """A request whose drafts are never accepted (yield 1) with a speculative cycle costing c
    plain steps: the controller spends `warmup` cycles, then decodes plainly, so N tokens take
    warmup * c + (N - warmup) steps, a speed of N / (N + warmup (c - 1)) of plain decode. With
    c = 1.4, warmup = 8 and N = 100 that is 0.969, the card's "about 0.96x" worst case."""
    c, warmup, N = 1.4, 8, 100
    flags, _ = _run([0] * N, break_even=c, warmup=warmup, window=8)
    time_steps, tokens, spec = 0.0, 0, True
    for f in flags:
        if tokens >= N:
            break
        time_steps += c if spec else 1.0
        tokens += 1
        spec = f
    assert tokens == N
    speed = N / time_steps
    assert speed == pytest.approx(N / (N + warmup * (c - 1)))
    assert 0.95 < speed < 0.97


def test_argument_errors_leave_the_state_unchanged(lib):
    q = bd.YieldQuench(2, 1.5)
    q.update(np.asarray([3, 3], np.int32))
    before = [q.state(b) for b in range(2)]
    for cfg in (bd.QuenchConfig(0.0, 8, 16, 0), bd.QuenchConfig(float("nan"), 8, 16, 0),
                bd.QuenchConfig(1.5, 0, 16, 0), bd.QuenchConfig(1.5, 8, 0, 0),
                bd.QuenchConfig(1.5, 8, bd.QUENCH_MAX_WINDOW + 1, 0),
                bd.QuenchConfig(1.5, 8, 16, -1)):
        out = np.zeros(2, np.int32)
        na = np.asarray([1, 1], np.int32)
        rc = lib.dspark_quench_update(ctypes.byref(cfg), ctypes.cast(q.states, ctypes.c_void_p),
                                      2, na.ctypes.data, None, out.ctypes.data)
        assert rc == 1
    with pytest.raises(bd.DsparkError):
        q.update(np.asarray([3, 33], np.int32))      # more accepted drafts than K can be
    assert [q.state(b) for b in range(2)] == before
    assert lib.dspark_quench_reset(None, -1) == 1
    assert lib.dspark_quench_update(ctypes.byref(q.config), None, 0, None, None, None) == 0
