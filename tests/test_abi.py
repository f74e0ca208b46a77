"""The C ABI without a GPU: the library builds, loads, exports what the header declares,
and rejects bad arguments synchronously, before any CUDA call."""

import ctypes

import pytest

from lossless_draft_verification_speculative_b200 import binding, build_lib

BF16, F32 = 0, 1
FAKE = 0x10000  # a 64 KiB-aligned fake device address: never dereferenced by these calls


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return binding.load_library()


def _out(n=FAKE, t=FAKE, nx=FAKE):
    return binding.AcceptOut(n, t, nx, None, None, None, None)


def test_exports_every_declared_symbol(lib):
    names = binding.header_functions()
    assert {"dspark_greedy_accept", "dspark_speculative_sample_accept",
            "dspark_workspace_bytes", "dspark_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert lib.dspark_status_string(code).decode() == name
    assert lib.dspark_status_string(99).decode() == "DSPARK_ERR_UNKNOWN"
    assert lib.dspark_version() >= 1


def test_workspace_bytes(lib):
    assert lib.dspark_workspace_bytes(64, 7, 129280, BF16) > 0
    assert lib.dspark_workspace_bytes(64, 7, 129280, BF16) < 8 << 20
    assert lib.dspark_workspace_bytes(1, 33, 100, BF16) == 0      # K > 32
    assert lib.dspark_workspace_bytes(1, 3, 0, BF16) == 0         # V < 1
    assert lib.dspark_workspace_bytes(1, 3, 262145, BF16) == 0    # V beyond the limit
    assert lib.dspark_workspace_bytes(1, 3, 64, 7) == 0           # unknown dtype
    a = lib.dspark_workspace_bytes(8, 7, 262144, BF16)
    b = lib.dspark_workspace_bytes(16, 7, 262144, BF16)
    assert b > a


def test_plans_cover_every_workload_shape(lib):
    for V in (1, 64, 2048, 2049, 129280, 151936, 262144):
        p = binding.Plan()
        assert lib.dspark_plan(4, 7, V, BF16, 1, ctypes.byref(p)) == 0
        assert p.n_chunks == -(-V // p.chunk_elems) and p.n_chunks * p.chunk_elems >= V
        assert p.elems_per_load == 8 and p.threads_per_cta % 32 == 0 and p.loads_in_flight >= 1
        assert p.stream_threads_per_cta % 32 == 0 and p.stream_threads_per_cta <= 1024
        # pass-1 units: one per (row, chunk); K+1 rows (greedy), 2K+1 rows (sampling)
        assert p.greedy_units_per_sequence == 8 * p.n_chunks
        assert p.sampling_units_per_sequence == 15 * p.n_chunks
        # one pass-2 cluster per sequence, one chunk per warp: 16-warp CTAs while the batch's
        # clusters fit on 148 SMs, else 32-warp CTAs
        for B in (4, 64, 200):
            q = binding.Plan()
            assert lib.dspark_plan(B, 7, V, BF16, 1, ctypes.byref(q)) == 0
            g16 = -(-q.n_chunks // 16)
            if B * g16 <= 148:
                assert q.finish_threads_per_cta == 512 and q.finish_ctas_per_sequence == g16 <= 8
            else:
                assert q.finish_threads_per_cta == 1024
                assert q.finish_ctas_per_sequence == -(-q.n_chunks // 32) <= 4
        assert lib.dspark_plan(4, 7, V, BF16, 0, ctypes.byref(p)) == 0
        assert p.elems_per_load == 1
        assert lib.dspark_plan(4, 7, V, F32, 1, ctypes.byref(p)) == 0
        assert p.elems_per_load == 4
    assert lib.dspark_plan(4, 7, 262145, BF16, 1, ctypes.byref(binding.Plan())) == 2


def test_workspace_needs_no_initialisation(lib):
    for B, K in ((1, 0), (64, 7), (256, 15), (3, 32)):
        assert lib.dspark_workspace_zero_bytes(B, K) == 0
        # one float2 record per (row, chunk) unit, 2K+1 rows per sequence, then the gathers
        nch = -(-129280 // 2048)
        assert lib.dspark_workspace_bytes(B, K, 129280, BF16) >= 8 * B * (2 * K + 1) * nch + 8 * B * K


def _greedy(lib, **kw):
    a = dict(p1=FAKE, ld=1024, pv=FAKE, ldv=7 * 1024, dt=BF16, d=FAKE, B=4, K=7, V=1024,
             out=_out(), ws=FAKE, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.dspark_greedy_accept(a["p1"], a["ld"], a["pv"], a["ldv"], a["dt"], a["d"], a["B"],
                                    a["K"], a["V"], a["out"], a["ws"], a["wsb"], a["s"])


def _sample(lib, **kw):
    a = dict(p1=FAKE, ld=1024, pv=FAKE, ldv=7 * 1024, q=FAKE, dt=BF16, d=FAKE, B=4, K=7, V=1024,
             T=1.0, u=FAKE, out=_out(), ws=FAKE, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.dspark_speculative_sample_accept(a["p1"], a["ld"], a["pv"], a["ldv"], a["q"], a["dt"],
                                                a["d"], a["B"], a["K"], a["V"], a["T"], a["u"],
                                                a["out"], a["ws"], a["wsb"], a["s"])


def _mixed(lib, **kw):
    a = dict(p1=FAKE, ld=1024, pv=FAKE, ldv=7 * 1024, q=FAKE, dt=BF16, d=FAKE, nd=FAKE, B=4, K=7,
             V=1024, T=FAKE, u=FAKE, out=_out(), ws=FAKE, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.dspark_mixed_accept(a["p1"], a["ld"], a["pv"], a["ldv"], a["q"], a["dt"], a["d"],
                                   a["nd"], a["B"], a["K"], a["V"], a["T"], a["u"], a["out"],
                                   a["ws"], a["wsb"], a["s"])


def _early_exit(lib, **kw):
    a = dict(p1=FAKE, ld=1024, pv=FAKE, ldv=7 * 1024, q=FAKE, dt=BF16, d=FAKE, B=4, K=7, V=1024,
             T=1.0, u=FAKE, out=_out(), ws=FAKE, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.dspark_early_exit_accept(a["p1"], a["ld"], a["pv"], a["ldv"], a["q"], a["dt"],
                                        a["d"], a["B"], a["K"], a["V"], a["T"], a["u"],
                                        a["out"], a["ws"], a["wsb"], a["s"])


@pytest.mark.parametrize("call", [_greedy, _sample, _mixed, _early_exit])
def test_invalid_arguments(lib, call):
    INV, UNS, WS = 1, 2, 4
    assert call(lib, B=-1) == INV
    assert call(lib, K=-1) == INV
    assert call(lib, K=33, ldv=33 * 1024) == INV
    assert call(lib, V=0) == INV
    assert call(lib, dt=5) == INV
    assert call(lib, p1=None) == INV
    assert call(lib, pv=None) == INV
    assert call(lib, d=None) == INV
    assert call(lib, ld=1000) == INV              # rows of p1 would overlap
    assert call(lib, ldv=6 * 1024) == INV         # sequences of pv would overlap
    assert call(lib, out=_out(n=None)) == INV
    assert call(lib, out=_out(t=None)) == INV
    assert call(lib, out=_out(nx=None)) == INV
    assert call(lib, p1=FAKE + 1) == UNS          # not aligned to the element size
    assert call(lib, V=262145, ld=262145, ldv=7 * 262145) == UNS
    assert call(lib, ld=1 << 31) == UNS           # row strides are 32-bit in the kernels
    assert call(lib, ldv=1 << 31) == UNS
    assert call(lib, ws=None) == WS
    assert call(lib, wsb=16) == WS
    assert call(lib, ws=FAKE + 16) == WS          # workspace must be 256-byte aligned
    assert call(lib, B=0) == 0                    # empty batch: a no-op


def test_sampling_specific_arguments(lib):
    INV, UNS = 1, 2
    assert _sample(lib, T=-0.5) == INV
    assert _sample(lib, T=float("nan")) == INV
    assert _sample(lib, T=float("inf")) == INV
    assert _sample(lib, T=1e-45) == INV           # log2(e)/T overflows float
    assert _sample(lib, q=None) == INV
    assert _sample(lib, u=None) == INV
    assert _sample(lib, q=FAKE + 1) == UNS
    # T == 0 is greedy_accept: q and uniforms are not needed, the greedy checks apply
    assert _sample(lib, T=0.0, q=None, u=None, ws=None) == 4
    # K == 0: no draft rows, pv / q / drafts may be NULL; workspace still checked
    assert _sample(lib, K=0, pv=None, q=None, d=None, ldv=0, ws=None) == 4


def test_mixed_batch_specific_arguments(lib):
    INV, UNS = 1, 2
    assert _mixed(lib, T=None) == INV             # temperatures are required
    assert _mixed(lib, u=None) == INV
    assert _mixed(lib, q=None) == INV             # required for K > 0 even if all are greedy
    assert _mixed(lib, q=FAKE + 1) == UNS
    # the draft counts may be NULL (every sequence K); the workspace check still applies
    assert _mixed(lib, nd=None, ws=None) == 4
    # K == 0: no draft rows; q and drafts may be NULL
    assert _mixed(lib, K=0, pv=None, q=None, d=None, ldv=0, ws=None) == 4


def test_markov_matvec_arguments(lib):
    INV, UNS = 1, 2
    mv = lambda t=FAKE, ty=0, V=1000, R=256, h=FAKE, B=1, y=FAKE: (  # noqa: E731
        lib.dspark_markov_matvec(t, ty, V, R, h, B, y, None))
    assert mv(ty=2) == INV
    assert mv(V=-1) == INV and mv(B=-1) == INV and mv(R=0) == INV
    assert mv(t=None) == INV and mv(h=None) == INV and mv(y=None) == INV
    assert mv(R=128) == UNS                        # the drafters ship rank 256
    assert mv(t=FAKE + 8) == UNS and mv(h=FAKE + 4) == UNS and mv(y=FAKE + 2) == UNS
    assert mv(V=0) == 0 and mv(B=0) == 0           # no-ops


def test_early_exit_specific_arguments(lib):
    INV, UNS, WS = 1, 2, 4
    assert _early_exit(lib, T=-0.5) == INV
    assert _early_exit(lib, T=float("nan")) == INV
    assert _early_exit(lib, T=1e-45) == INV
    assert _early_exit(lib, q=None) == INV
    assert _early_exit(lib, u=None) == INV
    assert _early_exit(lib, q=FAKE + 1) == UNS
    # T == 0 verifies greedily: q and uniforms may be NULL; the workspace check still applies
    assert _early_exit(lib, T=0.0, q=None, u=None, ws=None) == WS
    assert _early_exit(lib, K=0, pv=None, q=None, d=None, ldv=0, ws=None) == WS
    # the one workspace size serves every policy
    assert _early_exit(lib, wsb=lib.dspark_workspace_bytes(4, 7, 1024, BF16) - 1) == WS


def test_sample_pass1_arguments(lib):
    INV, UNS, WS = 1, 2, 4

    def p1(**kw):
        a = dict(p1=FAKE, ld=1024, pv=FAKE, ldv=7 * 1024, q=FAKE, dt=BF16, d=FAKE, B=4, K=7,
                 V=1024, T=1.0, ws=FAKE, wsb=1 << 30, s=None)
        a.update(kw)
        return lib.dspark_sample_pass1(a["p1"], a["ld"], a["pv"], a["ldv"], a["q"], a["dt"],
                                       a["d"], a["B"], a["K"], a["V"], a["T"], a["ws"], a["wsb"],
                                       a["s"])
    assert p1(T=0.0) == INV                       # no sampling pass at T == 0
    assert p1(T=float("nan")) == INV
    assert p1(q=None) == INV
    assert p1(B=-1) == INV
    assert p1(ld=1000) == INV
    assert p1(q=FAKE + 1) == UNS
    assert p1(ws=None) == WS
    assert p1(B=0) == 0
