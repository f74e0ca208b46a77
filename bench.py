"""Benchmark of the DSpark block verify step (greedy_accept + speculative_sample_accept).

One step = one verify call per temperature of the workload over one batch of B sequences:
for the DeepSeek-V4-Flash-shaped serving workload (B=64, K=7, V=129280, bf16) that is
greedy_accept (T=0), then speculative_sample_accept at T=0.7 and at T=1.0. Each call reads
a distinct copy of the inputs (4 rotating sets of ~248 MB, each larger than L2), so every
call streams its logits from HBM.

    python bench.py [--gpus N --steps K --warmup W]      # the CUDA path
    python bench.py --impl reference ...                  # the CPU float64 oracle

Under torchrun every rank verifies its own batch (B-sharded replicas, no collective); the
reported value is all ranks' verified blocks over the max-over-ranks device time.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "verified blocks/s and HBM GB/s vs B200 peak at B=64,K=7,V=129280 bf16"
FALLBACK_HBM_GBS = 6650.0
N_SETS = 4
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "stream_stats_kernel_dsv4_flash_serving.md")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dsv4_flash_serving")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="seconds of oracle work timed for the CPU baseline (whole steps)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-stress", action="store_true",
                    help="skip the early-exit timing on the B=256, K=15, V=262144 workload")
    return ap.parse_args()


def source_hash(files=("common.cuh", "stream.cuh")):
    """Hash of the sources a kernel is compiled from (default: the stream kernel's)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lossless_draft_verification_speculative_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """Per-launch DRAM bytes (read + write) of the sampling call's stream kernel from the
    committed ncu summary, if the kernel sources are unchanged since it was taken; else None."""
    try:
        kv = {}
        for line in open(PROFILE_SUMMARY):
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                v = v.strip()
                kv[k.strip()] = v.split("`")[1] if v.startswith("`") else v.split()[0]
        if kv.get("source_hash") != source_hash():
            return None
        return float(kv["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def rank_seed(rank: int) -> int:
    """Logit seed of a rank's batch: every rank verifies its own, distinct sequences."""
    from lossless_draft_verification_speculative_b200 import workloads as wl
    return wl.SEED_LOGITS + 1000 * rank


def aggregate(ms_local: float, blocks_per_rank: int, world: int, dist=None, device=None):
    """Whole-job throughput of B-sharded replicas: all ranks' verified blocks over the slowest
    rank's device time (max over ranks). Returns (blocks/s, max ms)."""
    import torch
    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    return blocks_per_rank * world / (ms_max / 1000.0), ms_max


def build_calls(w):
    return [("greedy" if T == 0 else "sample", float(T)) for T in w.temperatures]


# ------------------------------------------------------------------------- reference arm

def run_reference(args, w):
    """The oracle as it stands, on the host cores, on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from lossless_draft_verification_speculative_b200 import workloads as wl
    from oracle import accept_ref as ora

    calls = build_calls(w)
    # a step is one verified block: one sequence through one call, cycling through the
    # workload's temperatures and a pool of its sequences, so that any --steps ends in
    # minutes (about 12 ms of float64 work per block)
    pool = list(range(min(8, w.B)))
    P, Q = wl.logits(w, pool)
    Pf, Qf = wl.as_float64(P, w.dtype), wl.as_float64(Q, w.dtype)
    inputs = [(T, wl.drafts(w, Q, T, pool), wl.uniforms(w, pool, T=T).astype(np.float64))
              for _, T in calls]

    def step(s):
        T, d, u = inputs[s % len(calls)]
        b = (s // len(calls)) % len(pool)
        if T == 0:
            ora.greedy_accept(Pf[b:b + 1], d[b:b + 1])
        else:
            ora.speculative_sample_accept(Pf[b:b + 1], Qf[b:b + 1], d[b:b + 1], T, u[b:b + 1])

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(s)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    sample = (f"one block per step: sequence s//{len(calls)} mod {len(pool)} of the first "
              f"{len(pool)} of {w.B}, call s mod {len(calls)} (T={list(w.temperatures)}); "
              f"float64 NumPy, one process")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "blocks/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1000 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "K": w.K, "V": w.V,
                   "temperatures": list(w.temperatures), "blocks_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "blocks/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "blocks/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def cpu_baseline(w, seconds, outs=None):
    """The oracle timed on the host cores, and the bench's own results checked against it.

    Timings: on all host cores (one spawn-started process per core, at most one per sequence,
    each verifying its sequences through every call of the step over and over for `seconds`),
    and on one core (steps of 8 sequences through every call, repeated for `seconds`).
    Parity: with ``outs`` (the GPU results of the step's calls, rank 0's batch) every
    sequence of every call is compared with the oracle: greedy bit for bit, sampling decisions
    and tokens identical except where the oracle's uniform lies within 1e-6 of a boundary."""
    from oracle import parallel as par

    pool = par.timed_all_cores(w.name, w.temperatures, seconds)
    one = cpu_baseline_one_core(w, seconds)
    res = {"value": pool["value"], "unit": "blocks/s", "cores": pool["cores"], "kind": "oracle",
           "sample": f"{pool['blocks']} verified blocks ({w.B} sequences x {len(w.temperatures)} "
                     f"calls, repeated) in {pool['seconds']:.1f} s of float64 NumPy on "
                     f"{pool['cores']} processes, one per host core",
           "host_cores": par.host_cores(), "single_core": one}
    near = oracle_parity(w, outs) if outs is not None else None
    return res, near


def oracle_parity(w, outs):
    """Every sequence of the step's calls against the oracle (all host cores)."""
    from oracle import parallel as par

    calls = build_calls(w)
    per = {}
    total = {"sequences": 0, "near_boundary": 0, "differ": 0, "differ_outside_band": 0}
    for c, (kind, T) in enumerate(calls):
        o = par.run(w.name, T, seqs=range(w.B))
        n_g = outs[c].n_accepted.cpu().numpy()
        t_g = outs[c].tokens.cpu().numpy()
        same = (n_g == o["n_accepted"]) & np.all(t_g == o["tokens"], axis=1)
        near = o["near"] if kind == "sample" else np.zeros(w.B, bool)
        st = {"sequences": int(w.B), "near_boundary": int(near.sum()),
              "differ": int((~same).sum()), "differ_outside_band": int((~same & ~near).sum())}
        per[f"{kind}_T{T}"] = st
        for k in total:
            total[k] += st[k]
    total["calls"] = per
    total["eps"] = 1e-6
    return total


def cpu_baseline_one_core(w, seconds):
    """The oracle timed on one host core: steps of 8 sequences through every call of the
    workload, repeated until about `seconds` of work have run."""
    from lossless_draft_verification_speculative_b200 import workloads as wl
    from oracle import accept_ref as ora

    calls = build_calls(w)
    nseq = 8
    seqs = list(range(nseq))
    P, Q = wl.logits(w, seqs)
    Pf, Qf = wl.as_float64(P, w.dtype), wl.as_float64(Q, w.dtype)
    inputs = [(T, wl.drafts(w, Q, T, seqs), wl.uniforms(w, seqs, T=T).astype(np.float64))
              for _, T in calls]
    t0 = time.perf_counter()
    steps, dt = 0, 0.0
    while steps == 0 or dt < seconds:
        for T, d, u in inputs:
            if T == 0:
                ora.greedy_accept(Pf, d)
            else:
                ora.speculative_sample_accept(Pf, Qf, d, T, u)
        steps += 1
        dt = time.perf_counter() - t0
    blocks = steps * len(calls) * nseq
    return {"value": blocks / dt, "unit": "blocks/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps} x {len(calls)} calls x {nseq} of {w.B} sequences "
                      f"({dt:.1f} s of float64 NumPy on one host core)"}


# ----------------------------------------------------------------------------- our arm

def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import lossless_draft_verification_speculative_b200 as pkg
    from lossless_draft_verification_speculative_b200 import binding as bd
    from lossless_draft_verification_speculative_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    pkg.load_library()
    calls = build_calls(w)
    # inputs: this rank's own batch (distinct sequences per rank)
    P, Q, D = wl.generate(w, w.temperatures, seed=rank_seed(rank),
                          processes=min(16, os.cpu_count() or 1))
    U = {T: wl.uniforms(w, T=T) for T in w.temperatures}
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def host_tensor(a):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(a)

    Ph, Qh = host_tensor(P), host_tensor(Q)
    sets = []
    for s in range(N_SETS):
        if s == 0:
            sets.append((Ph.to(dev), Qh.to(dev)))
        else:
            sets.append((sets[0][0].clone(), sets[0][1].clone()))
    Dd = {T: torch.from_numpy(D[T]).to(dev) for T in w.temperatures}
    Ud = {T: torch.from_numpy(U[T]).to(dev) for T in w.temperatures}
    wsb = bd.workspace_bytes(w.B, w.K, w.V, tdt)
    workspace = bd.new_workspace(wsb, dev)
    outs = [bd._alloc_result(w.B, w.K, dev, diagnostics=(kind == "sample")) for kind, _ in calls]

    # one prepared call per (call, input set)
    prepared = []
    for c, (kind, T) in enumerate(calls):
        row = []
        for s in range(N_SETS):
            Pd, Qd = sets[s]
            row.append(bd.PreparedCall(kind, Pd, Qd, Dd[T], T, Ud[T], outs[c], workspace))
        prepared.append(row)
    ncalls = len(calls)

    def step(s):
        for c in range(ncalls):
            prepared[c][(s * ncalls + c) % N_SETS]()

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()

    # the timed region: K steps back to back, device time from two events around it
    clocks = ClockSampler(local) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for s in range(args.steps):
        step(s)
    t_end.record()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    barrier()
    ms = t_start.elapsed_time(t_end)

    # per call type: a run of back-to-back calls of that type alone (same rotating inputs),
    # events around the run; its mean is the call's duration on the device
    per_call_us = []
    reps = max(50, min(1000, args.steps))
    for c in range(ncalls):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for r in range(reps):
            prepared[c][r % N_SETS]()
        b.record()
        torch.cuda.synchronize()
        per_call_us.append(a.elapsed_time(b) * 1000.0 / reps)
    # the dominant kernel alone: pass 1 of each sampling call, back to back on the same inputs
    pass1_us = {}
    for c, (kind, T) in enumerate(calls):
        if kind == "sample":
            fns = [bd.PreparedCall("sample_pass1", Pd, Qd, Dd[T], T, Ud[T], outs[c], workspace)
                   for Pd, Qd in sets]
            pass1_us[T] = _time_calls(fns, reps)
    mixed = time_mixed_batch(w, sets, D, U, workspace, dev, reps)
    value, ms_max = aggregate(ms, args.steps * ncalls * w.B, world, dist, dev)

    # results of the last step: committed tokens per verified block
    committed = []
    for c in range(ncalls):
        committed.append(float((outs[c].n_accepted.double() + 1).mean().item()))

    # e2e: the public API with pinned host inputs, copies and the result read inside
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, calls, P, Q, D, U, dev, tdt, outs, workspace, world)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    # single-GPU characterisations beside the step, on the one-GPU line only (a scaling run
    # holds every GPU while rank 0 would run them)
    markov, small, early = {}, {}, {}
    if world == 1:
        markov = time_markov_matvec(dev)
        small = time_small_batches(dev)
        early = time_early_exit_serving(w, sets, Dd, Ud, workspace, dev, reps, per_call_us,
                                        calls)
        if not args.no_stress:
            early.update(time_early_exit_stress(dev))

    peaks = measured_peaks()
    peak = peaks["hbm_gbs"] if peaks else FALLBACK_HBM_GBS
    call_stats = {}
    samp_us = []
    for c, (kind, T) in enumerate(calls):
        us = per_call_us[c]
        nbytes = w.greedy_bytes() if kind == "greedy" else w.sampling_bytes()
        call_stats[f"{kind}_T{T}"] = {
            "us_per_call": us, "algorithmic_bytes": nbytes,
            "GB_per_s": nbytes / (us * 1e-6) / 1e9,
            "frac_of_peak": nbytes / (us * 1e-6) / 1e9 / peak,
            "committed_tokens_per_block": committed[c]}
        if kind == "sample":
            samp_us.append(us)
    samp_mean = statistics.mean(samp_us)
    call_achieved = w.sampling_bytes() / (samp_mean * 1e-6) / 1e9
    p1_mean = statistics.mean(pass1_us.values())
    achieved = w.sampling_bytes() / (p1_mean * 1e-6) / 1e9
    traffic = recorded_traffic()
    line = {
        "metric": METRIC, "value": value, "unit": "blocks/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "K": w.K, "V": w.V,
                   "temperatures": list(w.temperatures), "calls_per_step": ncalls,
                   "global_batch": w.B * world,
                   "l2": f"inputs larger than L2: {N_SETS} rotating input sets of "
                         f"{w.sampling_bytes() / 1e6:.1f} MB, a different set every call",
                   "parallelism": f"B-sharded replicas x{world}, no collective"},
        "gpu_launches": 2 * ncalls * args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "stream_stats_kernel<bf16, 8, sampling> (pass 1 of "
                               "speculative_sample_accept), launched alone through "
                               "dspark_sample_pass1, back to back on rotating inputs, mean over "
                               "the T>0 calls",
                     "us_per_launch": p1_mean,
                     "call_achieved": call_achieved, "call_frac": call_achieved / peak,
                     "call_us": samp_mean,
                     "call": "the whole sampling call (pass 1 + the finish), back to back",
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if peaks
                     else "fallback 6.65 TB/s"},
        "committed_token_equivalents_per_s": value * statistics.mean(committed),
        "calls": call_stats,
    }
    if mixed:
        mixed["frac_of_peak"] = mixed["GB_per_s"] / peak
        call_stats["mixed_batch"] = mixed
    if markov:
        for m in markov.values():
            m["frac_of_peak"] = m["GB_per_s"] / peak
        call_stats["markov_matvec"] = markov
    if early:
        call_stats["early_exit"] = early
    for m in small.values():
        m["frac_of_peak"] = m["GB_per_s"] / peak
    if small:
        call_stats["small_batches"] = small
    if clk:
        line["clocks"] = clk
    if e2e:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], near = cpu_baseline(w, args.cpu_seconds, outs)
        if near is not None:
            line["near_boundary"] = near
    print(json.dumps(line), flush=True)


def time_mixed_batch(w, sets, D, U, workspace, dev, reps):
    """A mixed serving batch on the same logits, timed alone (not part of the step): sequence
    b verifies K_b drafts at T_b (workloads.mixed_params), with the drafts and uniforms of the
    step's call at T_b. Its bytes are the rows it reads: P rows 0..K_b, and Q rows 0..K_b-1
    when T_b > 0."""
    import torch

    from lossless_draft_verification_speculative_b200 import binding as bd
    from lossless_draft_verification_speculative_b200 import workloads as wl

    kb, Tb = wl.mixed_params(w, w.temperatures)
    temps = np.asarray(w.temperatures, dtype=np.float64)
    ti = [int(np.argmin(np.abs(temps - float(t)))) for t in Tb]
    d = np.stack([D[w.temperatures[i]][b] for b, i in enumerate(ti)]).astype(np.int32)
    u = np.stack([U[w.temperatures[i]][b] for b, i in enumerate(ti)]).astype(np.float32)
    es = 2 if w.dtype == "bf16" else 4
    nbytes = int(sum(es * w.V * ((k + 1) + (k if t > 0 else 0)) for k, t in zip(kb, Tb)))
    kd, Td = torch.from_numpy(kb).to(dev), torch.from_numpy(Tb).to(dev)
    dd, ud = torch.from_numpy(d).to(dev), torch.from_numpy(u).to(dev)
    out = bd._alloc_result(w.B, w.K, dev, diagnostics=True)
    calls = [bd.PreparedCall("mixed", P, Q, dd, Td, ud, out, workspace, n_drafts=kd)
             for P, Q in sets]
    for r in range(8):
        calls[r % len(calls)]()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for r in range(reps):
        calls[r % len(calls)]()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1000.0 / reps
    return {"us_per_call": us, "bytes_read": nbytes, "GB_per_s": nbytes / (us * 1e-6) / 1e9,
            "mean_drafts": float(kb.mean()), "greedy_sequences": int((Tb == 0).sum()),
            "committed_tokens_per_block": float((out.n_accepted.double() + 1).mean().item())}


EE_BIG_PAIR_BYTES = 64 << 20  # the library's kEeBigPairBytes (early_exit.cuh)


def early_exit_waves(B, K, V, elem_bytes, sample):
    """The pairs [lo, hi) of each early-exit wave, as the library schedules them: waves of 1, 2,
    4, ... pairs when one row pair of the whole batch is at least 64 MB, else 2, 8, 32, ...,
    cut at K."""
    pair = B * V * elem_bytes * (2 if sample else 1)
    first, growth = (1, 2) if pair >= EE_BIG_PAIR_BYTES else (2, 4)
    waves, a, n = [], 0, first
    while True:
        lo, hi = min(a, K), min(a + n, K)
        waves.append((lo, hi))
        if hi >= K:
            return waves
        a, n = a + n, n * growth


def early_exit_bytes(n_accepted, K, V, elem_bytes, sample):
    """Bytes the early-exit call streams: each wave (``early_exit_waves``, the last adding the
    bonus row) reads its rows of every sequence that accepted all drafts before it, i.e. whose
    accepted count is at least the wave's first pair."""
    n = np.asarray(n_accepted)
    waves = early_exit_waves(n.size, K, V, elem_bytes, sample)
    rows = 0
    for i, (lo, hi) in enumerate(waves):
        per = (hi - lo) * (2 if sample else 1) + (1 if i == len(waves) - 1 else 0)
        rows += per * int((n >= lo).sum())
    return rows * V * elem_bytes


def _time_calls(fns, reps, warm=3):
    import torch

    for r in range(warm):
        fns[r % len(fns)]()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for r in range(reps):
        fns[r % len(fns)]()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) * 1000.0 / reps


def time_small_batches(dev, reps=300):
    """The two small verify workloads, timed alone (not part of the step): Qwen3-4B-shaped
    B=1, K=7, V=151936 and Gemma-4-12B-shaped B=8, K=7, V=262144, greedy and sampling at T=1,
    back-to-back calls on rotating copies of the inputs (more than L2 in all), so their
    latency floors (two dependent launches and the finish's chain) show beside the bytes."""
    import torch

    from lossless_draft_verification_speculative_b200 import binding as bd
    from lossless_draft_verification_speculative_b200 import workloads as wl

    res = {}
    for name in ("qwen3_4b_block7", "gemma4_12b_block7"):
        w = wl.WORKLOADS[name]
        P, Q = wl.logits(w)
        Pd = torch.from_numpy(P.view(np.int16)).to(dev).view(torch.bfloat16)
        Qd = torch.from_numpy(Q.view(np.int16)).to(dev).view(torch.bfloat16)
        copies = max(2, -(-200_000_000 // (Pd.numel() * 2 + Qd.numel() * 2)))
        sets = [(Pd, Qd)] + [(Pd.clone(), Qd.clone()) for _ in range(copies - 1)]
        ws = bd.new_workspace(bd.workspace_bytes(w.B, w.K, w.V, torch.bfloat16), dev)
        for T in (0.0, 1.0):
            dd = torch.from_numpy(wl.drafts(w, Q, T)).to(dev)
            ud = torch.from_numpy(wl.uniforms(w, T=T)).to(dev)
            out = bd._alloc_result(w.B, w.K, dev, diagnostics=True)
            kind = "greedy" if T == 0 else "sample"
            fns = [bd.PreparedCall(kind, p, q, dd, T, ud, out, ws) for p, q in sets]
            us = _time_calls(fns, reps, warm=len(fns))
            nb = w.greedy_bytes() if T == 0 else w.sampling_bytes()
            res[f"{name}_T{T}"] = {"us_per_call": us, "algorithmic_bytes": nb,
                                   "GB_per_s": nb / (us * 1e-6) / 1e9,
                                   "rotating_copies": copies}
        del sets, Pd, Qd, ws
    torch.cuda.empty_cache()
    return res


def time_early_exit_serving(w, sets, Dd, Ud, workspace, dev, reps, per_call_us, calls):
    """early_exit_accept on the step's inputs (outside the step), beside the full call of the
    same temperature: back-to-back calls on the rotating input sets. Bytes are those the
    waves stream (``early_exit_bytes``), from the call's own accepted counts."""
    from lossless_draft_verification_speculative_b200 import binding as bd

    res = {}
    for c, (kind, T) in enumerate(calls):
        out = bd._alloc_result(w.B, w.K, dev, diagnostics=True)
        fns = [bd.PreparedCall("early_exit", P, Q, Dd[T], T, Ud[T], out, workspace)
               for P, Q in sets]
        us = _time_calls(fns, reps)
        nb = early_exit_bytes(out.n_accepted.cpu().numpy(), w.K, w.V, w.elem_bytes, T > 0)
        res[f"{w.name}_T{T}"] = {"us_per_call": us, "full_call_us": per_call_us[c],
                                 "bytes_streamed": nb, "GB_per_s": nb / (us * 1e-6) / 1e9,
                                 "mean_accepted": float(out.n_accepted.double().mean().item())}
    return res


def time_early_exit_stress(dev, reps=20):
    """The B=256, K=15, V=262144 workload (4.2 GB per sampling call, far above L2): the full
    call and early_exit_accept at each of its temperatures, back to back on one input set."""
    import torch

    from lossless_draft_verification_speculative_b200 import binding as bd
    from lossless_draft_verification_speculative_b200 import workloads as wl

    w = wl.WORKLOADS["stress"]
    P, Q, D = wl.generate(w, w.temperatures, processes=min(16, os.cpu_count() or 1))
    Pd = torch.from_numpy(P.view(np.int16)).to(dev).view(torch.bfloat16)
    Qd = torch.from_numpy(Q.view(np.int16)).to(dev).view(torch.bfloat16)
    del P, Q
    ws = bd.new_workspace(bd.workspace_bytes(w.B, w.K, w.V, torch.bfloat16), dev)
    res = {}
    for T in w.temperatures:
        dd = torch.from_numpy(D[T]).to(dev)
        ud = torch.from_numpy(wl.uniforms(w, T=T)).to(dev)
        out_f = bd._alloc_result(w.B, w.K, dev, diagnostics=True)
        out_e = bd._alloc_result(w.B, w.K, dev, diagnostics=True)
        full = bd.PreparedCall("greedy" if T == 0 else "sample", Pd, Qd, dd, T, ud, out_f, ws)
        early = bd.PreparedCall("early_exit", Pd, Qd, dd, T, ud, out_e, ws)
        us_f = _time_calls([full], reps)
        us_e = _time_calls([early], reps)
        n = out_e.n_accepted.cpu().numpy()
        same = bool(torch.equal(out_f.tokens, out_e.tokens))
        full_bytes = w.greedy_bytes() if T == 0 else w.sampling_bytes()
        nb = early_exit_bytes(n, w.K, w.V, w.elem_bytes, T > 0)
        res[f"stress_T{T}"] = {"us_per_call": us_e, "full_call_us": us_f,
                               "full_call_bytes": full_bytes, "bytes_streamed": nb,
                               "GB_per_s": nb / (us_e * 1e-6) / 1e9,
                               "full_call_GB_per_s": full_bytes / (us_f * 1e-6) / 1e9,
                               "blocks_per_s": w.B / (us_e * 1e-6),
                               "full_call_blocks_per_s": w.B / (us_f * 1e-6),
                               "mean_accepted": float(n.mean()), "same_tokens": same}
    del Pd, Qd, ws
    torch.cuda.empty_cache()
    return res


MARKOV_V, MARKOV_R = 129280, 256  # the DSpark drafters' vocabulary and Markov rank


def time_markov_matvec(dev, n=50, replays=5):
    """The drafter's Markov-head table mat-vec (y = W h over a V x 256 table), timed alone (not
    part of the step): n calls on rotating copies of the table (more than L2 in total)
    captured in one CUDA graph, events around its replays. Bytes: the table, read once per
    call (the states and outputs are under 0.1% of it)."""
    import torch

    from lossless_draft_verification_speculative_b200 import binding as bd
    from lossless_draft_verification_speculative_b200 import workloads as wl

    res = {}
    stream = torch.cuda.Stream(device=dev)
    for fmt in ("f16", "q8_0"):
        raw = wl.markov_table(MARKOV_V, MARKOV_R, fmt)
        t0 = torch.from_numpy(raw.view(np.int16) if fmt == "f16" else raw).to(dev)
        nbytes = t0.numel() * t0.element_size()
        copies = -(-200_000_000 // nbytes)
        tabs = [t0] + [t0.clone() for _ in range(copies - 1)]
        for B in (1, 4, 8, 64):
            h = torch.from_numpy(wl.markov_states(B, MARKOV_R)).to(dev)
            y = torch.empty(B, MARKOV_V, device=dev)
            with torch.cuda.stream(stream):
                for i in range(8):
                    bd.markov_matvec(tabs[i % copies], fmt, h, out=y)
            torch.cuda.synchronize(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    bd.markov_matvec(tabs[i % copies], fmt, h, out=y)
            for _ in range(3):
                g.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            a.record()
            for _ in range(replays):
                g.replay()
            b.record()
            torch.cuda.synchronize(dev)
            us = a.elapsed_time(b) * 1000.0 / (replays * n)
            res[f"{fmt}_B{B}"] = {"us_per_call": us, "table_bytes": nbytes,
                                  "GB_per_s": nbytes / (us * 1e-6) / 1e9}
            del g
        del tabs, t0
    return res


def run_e2e(args, w, calls, P, Q, D, U, dev, tdt, outs, workspace, world):
    import torch
    import torch.distributed as dist
    import lossless_draft_verification_speculative_b200 as pkg

    def pinned(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16) \
            if dt == "bf16" else torch.from_numpy(np.ascontiguousarray(a))
        return t.pin_memory()

    Ph, Qh = pinned(P, w.dtype), pinned(Q, w.dtype)
    Dh = {T: pinned(D[T]) for T in w.temperatures}
    Uh = {T: pinned(U[T]) for T in w.temperatures}
    Pd = torch.empty(Ph.shape, dtype=tdt, device=dev)
    Qd = torch.empty(Qh.shape, dtype=tdt, device=dev)
    Dd = {T: torch.empty_like(Dh[T], device=dev) for T in w.temperatures}
    Ud = {T: torch.empty_like(Uh[T], device=dev) for T in w.temperatures}
    res_h = [(torch.empty(w.B, dtype=torch.int32).pin_memory(),
              torch.empty(w.B, w.K + 1, dtype=torch.int32).pin_memory()) for _ in calls]
    h2d = 0
    d2h = 0
    for kind, T in calls:
        h2d += Ph.numel() * Ph.element_size() + Dh[T].numel() * 4
        if kind == "sample":
            h2d += Qh.numel() * Qh.element_size() + Uh[T].numel() * 4
        d2h += w.B * 4 + w.B * (w.K + 1) * 4

    def step():
        for c, (kind, T) in enumerate(calls):
            Pd.copy_(Ph, non_blocking=True)
            Dd[T].copy_(Dh[T], non_blocking=True)
            if kind == "greedy":
                r = pkg.greedy_accept(Pd, Dd[T], out=outs[c], workspace=workspace)
            else:
                Qd.copy_(Qh, non_blocking=True)
                Ud[T].copy_(Uh[T], non_blocking=True)
                r = pkg.speculative_sample_accept(Pd, Qd, Dd[T], T, Ud[T], out=outs[c],
                                                  workspace=workspace)
            res_h[c][0].copy_(r.n_accepted, non_blocking=True)
            res_h[c][1].copy_(r.tokens, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.e2e_steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = torch.tensor([t0.elapsed_time(t1)], device=dev, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    blocks = args.e2e_steps * len(calls) * w.B * world
    return {"value": blocks / (float(ms.item()) / 1000), "unit": "blocks/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": float(ms.item()) / args.e2e_steps}


def main():
    args = parse_args()
    from lossless_draft_verification_speculative_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
