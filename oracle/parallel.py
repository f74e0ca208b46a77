"""The CPU oracle run over many sequences or cycles of a seeded workload, on all host cores.

TEST INFRASTRUCTURE. Like ``accept_ref``, only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arms may import or run this module.

It adds no arithmetic of its own: each worker process regenerates its share of the inputs
from the seeded generators (``workloads``; every sequence and every cycle has its own
generator, so any subset can be rebuilt alone) and calls ``accept_ref`` on them, one
sequence (or cycle) at a time, exactly as a single process would. Workers are started with
``spawn``, so a caller that already holds a CUDA context can use it safely.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import time
from typing import Dict, List, Optional, Sequence

import numpy as np

FIELDS = ("n_accepted", "tokens", "next_token", "status", "p_draft", "q_draft", "resid_mass",
          "accept_margin", "cdf_margin", "near")


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _single_thread_env():
    for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[k] = "1"


def _inputs(name: str, mode: str, idx: Sequence[int], T: float, seed: int):
    """(P, Q, drafts, uniforms) for sequences ``idx`` (mode "seqs") or for cycles ``idx`` of
    sequence 0's fixed logits (mode "cycles"), stored form (bf16 bits or float32)."""
    from lossless_draft_verification_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    if mode == "seqs":
        P, Q = wl.logits(w, idx, seed)
        return P, Q, wl.drafts(w, Q, T, idx), wl.uniforms(w, idx, T=T)
    P1, Q1 = wl.logits(w, [0], seed)
    d = np.concatenate([wl.drafts(w, Q1, T, [0], cycle=c) for c in idx])
    u = np.concatenate([wl.uniforms(w, [0], T=T, cycle=c) for c in idx])
    return P1, Q1, d, u


def _verify(name: str, P, Q, d, u, T: float, shared: bool):
    """accept_ref on each row of (d, u) in turn; ``shared``: every row uses P[0], Q[0]."""
    from lossless_draft_verification_speculative_b200 import workloads as wl

    from . import accept_ref as ora

    w = wl.WORKLOADS[name]
    n, K = d.shape
    out = {"n_accepted": np.zeros(n, np.int32), "tokens": np.zeros((n, K + 1), np.int32),
           "next_token": np.zeros(n, np.int32), "status": np.zeros(n, np.int32),
           "p_draft": np.full((n, K), np.nan), "q_draft": np.full((n, K), np.nan),
           "resid_mass": np.full(n, np.nan), "accept_margin": np.full((n, K), np.inf),
           "cdf_margin": np.full(n, np.inf), "near": np.zeros(n, bool)}
    for k in range(n):
        s = 0 if shared else k
        Pf = wl.as_float64(P[s:s + 1], w.dtype)
        if T == 0:
            r = ora.greedy_accept(Pf, d[k:k + 1])
        else:
            r = ora.speculative_sample_accept(Pf, wl.as_float64(Q[s:s + 1], w.dtype),
                                              d[k:k + 1], T, u[k:k + 1].astype(np.float64))
            out["p_draft"][k], out["q_draft"][k] = r.p_draft[0], r.q_draft[0]
            out["resid_mass"][k] = r.resid_mass[0]
            out["accept_margin"][k], out["cdf_margin"][k] = r.accept_margin[0], r.cdf_margin[0]
            out["near"][k] = r.near_boundary()[0]
        out["n_accepted"][k], out["tokens"][k] = r.n_accepted[0], r.tokens[0]
        out["next_token"][k], out["status"][k] = r.next_token[0], r.status[0]
    return out


def _task(args):
    name, mode, idx, T, seed = args
    P, Q, d, u = _inputs(name, mode, idx, T, seed)
    res = _verify(name, P, Q, d, u, T, shared=(mode == "cycles"))
    res["drafts"], res["uniforms"] = d, u
    return res


def run(name: str, T: float, seqs: Optional[Sequence[int]] = None,
        cycles: Optional[Sequence[int]] = None, seed: int = 0,
        processes: Optional[int] = None) -> Dict[str, np.ndarray]:
    """The oracle's results for sequences ``seqs`` (or cycles ``cycles`` of sequence 0's fixed
    logits) of workload ``name`` at temperature T, in order, with the drafts and uniforms it
    used. Keys: FIELDS plus "drafts", "uniforms"; "near" marks the sequences whose uniforms
    lie within 1e-6 of a decision or CDF boundary (``OracleResult.near_boundary``)."""
    mode = "cycles" if cycles is not None else "seqs"
    idx = list(cycles if cycles is not None else seqs)
    procs = max(1, min(processes or host_cores(), len(idx)))
    parts = [idx[k::procs] for k in range(procs)]
    tasks = [(name, mode, p, float(T), seed) for p in parts if p]
    if len(tasks) == 1:
        results = [_task(tasks[0])]
    else:
        _single_thread_env()
        with mp.get_context("spawn").Pool(len(tasks)) as pool:
            results = pool.map(_task, tasks)
    # part k holds positions k, k + procs, ... of idx
    out = {}
    for key, first in results[0].items():
        arr = np.empty((len(idx),) + first.shape[1:], dtype=first.dtype)
        for k, r in enumerate(results):
            arr[k::procs] = r[key]
        out[key] = arr
    return out


def as_result(res: Dict[str, np.ndarray], T: float):
    """The dict of ``run`` as an ``accept_ref.OracleResult``."""
    from .accept_ref import OracleResult

    keys = ["n_accepted", "tokens", "next_token", "status"]
    if T > 0:
        keys += ["p_draft", "q_draft", "resid_mass", "accept_margin", "cdf_margin"]
    return OracleResult(**{k: res[k] for k in keys})


# ---------------------------------------------------------------- timed, all host cores

def _timed_worker(name, seqs, temps, seed, seconds, barrier, queue):
    _single_thread_env()
    from lossless_draft_verification_speculative_b200 import workloads as wl

    from . import accept_ref as ora

    w = wl.WORKLOADS[name]
    P, Q = wl.logits(w, seqs, seed)
    Pf, Qf = wl.as_float64(P, w.dtype), wl.as_float64(Q, w.dtype)
    calls = [(T, wl.drafts(w, Q, T, seqs), wl.uniforms(w, seqs, T=T).astype(np.float64))
             for T in temps]
    barrier.wait()
    t0 = time.perf_counter()
    blocks = 0
    while True:
        for T, d, u in calls:
            for k in range(len(seqs)):
                if T == 0:
                    ora.greedy_accept(Pf[k:k + 1], d[k:k + 1])
                else:
                    ora.speculative_sample_accept(Pf[k:k + 1], Qf[k:k + 1], d[k:k + 1], T,
                                                  u[k:k + 1])
                blocks += 1
        if time.perf_counter() - t0 >= seconds:
            break
    queue.put((blocks, time.perf_counter() - t0))


def timed_all_cores(name: str, temps: Sequence[float], seconds: float, seed: int = 0,
                    processes: Optional[int] = None) -> dict:
    """The oracle's throughput on all host cores: one spawn-started process per core (at
    most one per sequence), each owning the sequences b = k mod n, building their inputs,
    then, from a common start, verifying each of them through every call of ``temps`` over
    and over for at least ``seconds``. Returns blocks/s over the wall time from the start to
    the last process's end, and the process count."""
    from lossless_draft_verification_speculative_b200 import workloads as wl

    w = wl.WORKLOADS[name]
    n = max(1, min(processes or host_cores(), w.B))
    ctx = mp.get_context("spawn")
    _single_thread_env()
    barrier = ctx.Barrier(n + 1)
    queue = ctx.Queue()
    procs: List = []
    for k in range(n):
        seqs = list(range(k, w.B, n))
        p = ctx.Process(target=_timed_worker,
                        args=(name, seqs, list(temps), seed, seconds, barrier, queue))
        p.start()
        procs.append(p)
    barrier.wait()
    t0 = time.perf_counter()
    got = [queue.get() for _ in range(n)]
    wall = time.perf_counter() - t0
    for p in procs:
        p.join()
    blocks = sum(b for b, _ in got)
    return {"value": blocks / wall, "cores": n, "blocks": blocks, "seconds": wall}
