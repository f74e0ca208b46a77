"""The sampling call gives the oracle's results under every launch geometry.

Pass 1 splits the units over the grid by a fixed rule (CTA k takes units k, k + grid, ...),
so its records, and everything after them, must not depend on the grid size: a single CTA
(whose warps then stream every unit), three CTAs, an odd 37 (units of a sequence fall on the
CTAs unevenly) and the default one per SM all must give the same results. The cases cover
ragged vocabularies, K = 0 and K = 32, a 262144-token vocabulary, many short rows, and the
greedy policy.
"""

import numpy as np
import pytest
import torch

from lossless_draft_verification_speculative_b200 import binding as bd
from lossless_draft_verification_speculative_b200 import workloads as wl

from gpu_helpers import DEV, compare_greedy, compare_sampling, run_oracle, to_dev

pytestmark = pytest.mark.gpu

SCHEDULES = {
    "default": {},
    "grid1": {"DSPARK_MAX_CTAS": "1"},
    "grid3": {"DSPARK_MAX_CTAS": "3"},
    "grid37": {"DSPARK_MAX_CTAS": "37"},
}


def _run(P, Q, d, u, T, dtype, ws):
    Pd, Qd = to_dev(P, dtype), (to_dev(Q, dtype) if d.shape[1] else None)
    dd = torch.from_numpy(np.ascontiguousarray(d, dtype=np.int32)).to(DEV)
    ud = torch.from_numpy(np.ascontiguousarray(u, dtype=np.float32)).to(DEV)
    if T == 0:
        r = bd.greedy_accept(Pd, dd, workspace=ws)
    else:
        r = bd.speculative_sample_accept(Pd, Qd, dd, T, ud, workspace=ws)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in vars(r).items() if v is not None}


def _case(name, B, K, V, dtype, kind, params, T, ws, label):
    w = wl.Workload(name, B=B, K=K, V=V, dtype=dtype, kind=kind, params=params)
    P, Q = wl.logits(w)
    d = wl.drafts(w, Q, T)
    u = wl.uniforms(w, T=T)
    g = _run(P, Q, d, u, T, dtype, ws)
    o = run_oracle(P, Q, d, u, T, dtype)
    if T == 0:
        compare_greedy(g, o)
        return 0
    return compare_sampling(g, o, label, (P, Q, u, T, dtype))


CASES = [
    # name, B, K, V, dtype, kind, params, T
    ("serving", 64, 7, 129280, "bf16", "shared_noise", {"sd": 3.0, "noise": 1.0}, 1.0),
    ("ragged", 9, 5, 4097, "f32", "iid", {"sd": 2.0}, 0.8),
    ("k0", 6, 0, 5000, "bf16", "iid", {"sd": 2.0}, 1.0),
    ("k32", 3, 32, 3000, "bf16", "shared_noise", {"sd": 2.0, "noise": 0.5}, 1.0),
    ("wide", 2, 7, 262144, "bf16", "shared_noise", {"sd": 4.0, "noise": 0.5}, 1.3),
    ("many", 300, 3, 64, "f32", "iid", {"sd": 2.0}, 1.0),
    ("serving_greedy", 64, 7, 129280, "bf16", "shared_noise", {"sd": 3.0, "noise": 1.0}, 0.0),
    ("ragged_greedy", 9, 5, 4097, "f32", "iid", {"sd": 2.0}, 0.0),
]


@pytest.mark.parametrize("sched", list(SCHEDULES))
def test_schedules_agree_with_oracle(sched, monkeypatch):
    for k, v in SCHEDULES[sched].items():
        monkeypatch.setenv(k, v)
    nb = max(bd.workspace_bytes(c[1], c[2], c[3], torch.bfloat16 if c[4] == "bf16" else
                                torch.float32) for c in CASES)
    ws = bd.new_workspace(nb, DEV)
    near = 0
    for c in CASES:
        near += _case(*c, ws=ws, label=f"{sched}:{c[0]}")
    assert near <= 10


def test_calls_of_alternating_sizes():
    """Calls whose finish kernel needs more, then less, then more shared memory (the number of
    chunks per CTA follows V), and batches that grow and shrink: each call must be right
    whatever ran before it in the process."""
    for B, V in ((2, 9000), (64, 262144), (3, 4096), (300, 70000), (5, 262144), (64, 9000)):
        w = wl.Workload("alt", B=B, K=3, V=V, dtype="bf16", kind="iid", params={"sd": 2.0})
        P, Q = wl.logits(w)
        d = wl.drafts(w, Q, 1.0)
        u = wl.uniforms(w, T=1.0)
        ws = bd.new_workspace(bd.workspace_bytes(B, 3, V, torch.bfloat16), DEV)
        compare_sampling(_run(P, Q, d, u, 1.0, "bf16", ws), run_oracle(P, Q, d, u, 1.0, "bf16"),
                         f"alt B={B} V={V}", (P, Q, u, 1.0, "bf16"))


@pytest.mark.parametrize("V,dtype", [(129280, "bf16"), (5001, "f32")])
def test_pass1_alone_writes_the_full_calls_records(V, dtype):
    """dspark_sample_pass1 (the benchmark's timing of the dominant kernel) launches the same
    pass 1 as a full sampling call: the records and gathered logits in the workspace match
    bit for bit."""
    w = wl.Workload("p1", B=16, K=7, V=V, dtype=dtype, kind="mixed_sigma",
                    params={"sd": 3.0, "sigmas": (0.25, 1.0, 4.0)})
    P, Q = wl.logits(w)
    T = 0.7
    d, u = wl.drafts(w, Q, T), wl.uniforms(w, T=T)
    Pd, Qd = to_dev(P, dtype), to_dev(Q, dtype)
    dd = torch.from_numpy(d).to(DEV)
    ud = torch.from_numpy(u).to(DEV)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    nb = bd.workspace_bytes(w.B, w.K, w.V, tdt)
    ws_full, ws_p1 = bd.new_workspace(nb, DEV), bd.new_workspace(nb, DEV)
    bd.speculative_sample_accept(Pd, Qd, dd, T, ud, workspace=ws_full)
    out = bd._alloc_result(w.B, w.K, DEV, diagnostics=True)
    bd.PreparedCall("sample_pass1", Pd, Qd, dd, T, ud, out, ws_p1)()
    torch.cuda.synchronize()
    nch = -(-V // 2048)
    rec = w.B * (2 * w.K + 1) * nch * 8
    gat0 = -(-rec // 256) * 256
    assert torch.equal(ws_full[:rec], ws_p1[:rec])
    assert torch.equal(ws_full[gat0:gat0 + w.B * w.K * 8], ws_p1[gat0:gat0 + w.B * w.K * 8])
