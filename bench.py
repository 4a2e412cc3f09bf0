#!/usr/bin/env python
"""Benchmark of librlscan: env-steps/s per estimator and fraction of the B200
HBM roofline, on the sequence-length sweep N = 4096, T = 32..2048.

One *step* is one pass of the whole hot path over one batch of synthetic
rollouts: every estimator of the workload at every T of the sweep (the
default workload: GAE, V-trace, TD(lambda) and discounted returns at
T = 32, 64, ..., 2048 with per-step truncation -- 28 fused kernel launches).
Inputs are resident in HBM before the timed region; every call reads its own
buffers, so a step touches ~1.1 GB of distinct inputs (8.5x the 126 MB L2)
and no call finds its inputs in L2.  Steps are replayed from CUDA graphs;
timing-event nodes between launches give each kernel's duration on the
launching stream.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        python bench.py --impl reference ...     (the fp64 CPU oracle, timed)
Under torchrun each rank processes its own rollout shard of the workload
(weak scaling, no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from segmented_linear_recurrence_b200 import synthetic  # noqa: E402

METRIC = "env-steps/sec per estimator and % of B200 HBM roofline, N=4096, T=32..2048"
UNIT = "env-steps/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "sweep_4096xT"

# Bytes per env-step each estimator must move at minimum (mandatory inputs
# read once, outputs written once): fp32/int32 = 4 B, flags = 1 B.
def algorithmic_bytes(est: str, d: dict, real_bytes: int = 4) -> int:
    """Strict algorithmic HBM bytes of one call on inputs `d`.

    Per-step arrays count their full size; `truncated` adds its flag bytes and
    `trunc_value` is counted only where truncated (one 32-byte sector each);
    per-row arrays (bootstrap, init_trace) count one element per row; every
    output counts one element per step.  `real_bytes` is the size of a real
    element: 4 (fp32), or 2 for bf16 I/O."""
    if est == "affine_scan":  # a, b, reset flags, init per row, one output
        N, T = d["a"].shape
        return int(8 * N * T + (N * T if d.get("reset") is not None else 0)
                   + (4 * N if d.get("init") is not None else 0) + 4 * N * T)
    if est == "retrace":
        N, T, A = d["q"].shape
    else:
        key = {"elig_trace": "inputs", "episodic_prefix_sum": "x"}.get(est, "rewards")
        N, T = d[key].shape
        A = 0
    nt = N * T
    per_step_in = {
        "gae": ("rewards", "values"), "td_lambda": ("rewards", "values"),
        "vtrace": ("log_rhos", "rewards", "values"), "discounted_return": ("rewards",),
        "elig_trace": ("inputs",), "episodic_prefix_sum": ("x",),
        "retrace": ("mu_a", "actions", "rewards"),
    }[est]
    rb = real_bytes
    b = sum((4 if k == "actions" else rb) * nt for k in per_step_in)
    if est == "retrace":
        b += 2 * 4 * nt * A  # q and pi
    if d.get("terminated") is not None:
        b += nt
    if d.get("truncated") is not None:
        b += nt
        if d.get("trunc_value") is not None:
            b += 32 * int(np.count_nonzero(d["truncated"]))
    for k in ("bootstrap", "init_trace"):
        if d.get(k) is not None:
            b += rb * N
    n_out = {"gae": 2, "vtrace": 2}.get(est, 1)
    b += (4 if est == "episodic_prefix_sum" else rb) * nt * n_out
    return int(b)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(workload: str, est: str):
    """Per-launch DRAM bytes of one estimator's kernel in a workload, from the
    committed ncu summary, if it was taken on the current kernel sources (else
    None)."""
    from segmented_linear_recurrence_b200 import build as slr_build
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
    except Exception:
        return None
    if j.get("source_hash") != slr_build.source_hash():
        return None
    k = j.get("workloads", {}).get(workload, {}).get("kernels", {}).get(est)
    return None if k is None else k.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# multi-rank host logic (weak scaling over independent env shards)
# ---------------------------------------------------------------------------
def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own rollout shard: same shapes, different data."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank device-timed duration over all ranks (no-op alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_rank: int, max_ms: float) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1000.0)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
ARG_ORDER = {
    "gae": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
    "vtrace": ("log_rhos", "rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
    "retrace": ("q", "pi", "mu_a", "actions", "rewards", "bootstrap", "terminated", "truncated",
                "trunc_value"),
    "td_lambda": ("rewards", "values", "bootstrap", "terminated", "truncated", "trunc_value"),
    "discounted_return": ("rewards", "bootstrap", "terminated", "truncated", "trunc_value"),
    "elig_trace": ("inputs", "init_trace", "terminated", "truncated"),
    "episodic_prefix_sum": ("x", "terminated", "truncated"),
    "affine_scan": ("a", "b", "reset", "init"),
}
OUT_KW = {"gae": ("advantages", "returns"), "vtrace": ("vs", "pg_advantages"), "retrace": ("q_ret",),
          "td_lambda": ("returns",), "discounted_return": ("returns",), "elig_trace": ("traces",),
          "episodic_prefix_sum": ("out",), "affine_scan": ("x",)}


def workload_calls(workload: str, rank: int):
    """Host inputs of every call of one step: list of (est, T, dict)."""
    w = synthetic.WORKLOADS[workload]
    calls = []
    for est in w["estimators"]:
        for T in w["Ts"]:
            seed = shard_seed(synthetic.seed_for(workload, est, T), rank)
            if est == "affine_scan":
                d = synthetic.make_affine_inputs(w["N"], T, seed=seed, p_reset=w["p_term"])
            else:
                d = synthetic.make_inputs(est, w["N"], T, seed=seed, p_term=w["p_term"],
                                          p_trunc=w["p_trunc"], A=w.get("A", 18))
            calls.append((est, T, d))
    return calls


def time_major(workload: str) -> bool:
    return synthetic.WORKLOADS[workload].get("layout") == "time_major"


def bf16_io(workload: str) -> bool:
    return synthetic.WORKLOADS[workload].get("io") == "bf16"


REAL_KEYS = ("rewards", "values", "bootstrap", "trunc_value")  # the arrays bf16 I/O stores as bfloat16


def call_arrays(est, d, tm):
    """The call's input arrays in argument order, time-major when `tm`."""
    dd = synthetic.to_time_major(d) if tm else d
    return [dd.get(k) for k in ARG_ORDER[est]]


def call_plan(slr, est, d, T, tm):
    A = d["q"].shape[2] if est == "retrace" else 1
    N = d["q"].shape[0] if est == "retrace" else d[ARG_ORDER[est][0]].shape[0]
    return slr.rlscan_query_plan_tm(est, N, T) if tm else slr.rlscan_query_plan(est, N, T, A)


class DeviceCall:
    def __init__(self, est, T, d, device, tm=False, bf16=False):
        import torch
        self.est, self.T, self.tm, self.bf16 = est, T, tm, bf16
        self.inputs = []
        for k, a in zip(ARG_ORDER[est], call_arrays(est, d, tm)):
            t = None if a is None else torch.from_numpy(a).to(device)
            if t is not None and bf16 and k in REAL_KEYS:
                t = t.to(torch.bfloat16)
            self.inputs.append(t)
        shape = d["q"].shape[:2] if est == "retrace" else d[ARG_ORDER[est][0]].shape
        shape = tuple(shape[::-1]) if tm else tuple(shape)
        dt = torch.int32 if est == "episodic_prefix_sum" else (torch.bfloat16 if bf16 else torch.float32)
        self.outs = {k: torch.empty(shape, dtype=dt, device=device) for k in OUT_KW[est]}
        self.scal = {} if est == "episodic_prefix_sum" else dict(synthetic.SCALARS[est])
        self.steps = int(np.prod(shape))
        self.bytes = algorithmic_bytes(est, d, 2 if bf16 else 4)
        self.fn = f"rlscan_{est}{'_tm' if tm else ''}{'_bf16' if bf16 else ''}"

    def launch(self):
        import segmented_linear_recurrence_b200 as slr
        getattr(slr, self.fn)(*self.inputs, **self.scal, **self.outs)


def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import segmented_linear_recurrence_b200 as slr
    from segmented_linear_recurrence_b200 import build as slr_build

    slr_build.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)

    host_calls = workload_calls(args.workload, rank)
    tm = time_major(args.workload)
    calls = [DeviceCall(est, T, d, device, tm, bf16_io(args.workload)) for est, T, d in host_calls]
    steps_per_step = sum(c.steps for c in calls)
    launches_per_step = 0
    for est, T, d in host_calls:
        launches_per_step += call_plan(slr, est, d, T, tm)["launches"]

    def eager_step():
        for c in calls:
            c.launch()

    # warm-up: one eager step on the capture stream (so its workspace exists
    # before capture), then graph replays
    cap_stream = torch.cuda.Stream(device)
    ws = 0
    for est, T, d in host_calls:
        ws = max(ws, call_plan(slr, est, d, T, tm)["workspace_bytes"])
    slr.rlscan_reserve_workspace(ws, cap_stream)
    warm_done = 0
    with torch.cuda.stream(cap_stream):
        eager_step()
    warm_done += 1
    torch.cuda.synchronize()
    if slr.rlscan_sync_status() != 0:
        raise RuntimeError("device status error during warm-up")

    def capture(marks):
        """A graph of one step; `marks` = indices of calls preceded by a timing event
        (plus one event after the last call).  Returns (graph, events)."""
        g = torch.cuda.CUDAGraph()
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(marks) + 1)]
        with torch.cuda.graph(g, stream=cap_stream):
            cur = torch.cuda.current_stream()
            e = 0
            for j, c in enumerate(calls):
                if e < len(marks) and marks[e] == j:
                    evs[e].record(cur)
                    e += 1
                c.launch()
            evs[-1].record(cur)
        return g, evs

    # Concurrent step graph: the workload's calls are independent, so each
    # estimator's calls run on a stream of their own (fork from and join back
    # to the capture stream); every stream has its own look-back workspace.
    ests = list(dict.fromkeys(c.est for c in calls))
    nstreams = max(1, min(args.streams, len(ests)))
    side = [torch.cuda.Stream(device) for _ in range(nstreams)] if nstreams > 1 else []
    for s_ in side:
        slr.rlscan_reserve_workspace(ws, s_)

    def launch_concurrent(root):
        for s_ in side:
            s_.wait_stream(root)
        for j, c in enumerate(calls):
            with torch.cuda.stream(side[ests.index(c.est) % nstreams]):
                c.launch()
        for s_ in side:
            root.wait_stream(s_)

    g_conc = None
    if side:
        launch_concurrent(cap_stream)  # eager once: each stream's workspace in use before capture
        torch.cuda.synchronize()
        g_conc = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_conc, stream=cap_stream):
            launch_concurrent(torch.cuda.current_stream())

    # plain step graph (timed: value), per-estimator-group events (timed:
    # roofline), per-launch events (diagnostic per-T table)
    g_plain, _ = capture([])
    groups = []
    for j, c in enumerate(calls):
        if j == 0 or calls[j - 1].est != c.est:
            groups.append(j)
    g_group, ev_group = capture(groups)
    g_each, ev_each = capture(list(range(len(calls))))
    while warm_done < max(args.warmup, 1):
        (g_conc or g_plain).replay()
        warm_done += 1
    if g_conc is not None:
        g_plain.replay()
    g_group.replay()
    g_each.replay()
    torch.cuda.synchronize()

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(gpu_uuid)
    time.sleep(0.3)  # let the sampler start before the timed region

    def timed(graph, per_step_events=None):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        acc = None if per_step_events is None else np.zeros(len(per_step_events) - 1)
        t0.record(stream)
        for k in range(args.steps):
            graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        if per_step_events is not None:  # the last replay's intervals
            acc = np.array([per_step_events[i].elapsed_time(per_step_events[i + 1])
                            for i in range(len(per_step_events) - 1)])
        return t0.elapsed_time(t1), acc

    serial_ms, _ = timed(g_plain)
    elapsed_ms = timed(g_conc)[0] if g_conc is not None else serial_ms
    group_ms_total, group_last = timed(g_group, ev_group)
    clocks = sampler.stop()
    _, each_last = timed(g_each, ev_each)
    status = slr.rlscan_sync_status()
    # per-group time averaged over the whole group-timed region: scale the last
    # replay's split by the region's total
    group_ms = group_last * (group_ms_total / args.steps) / max(group_last.sum(), 1e-9)
    per_group = {calls[j].est: float(group_ms[i]) for i, j in enumerate(groups)}
    per_call_ms = each_last
    del g_plain, g_group, g_each, g_conc
    max_ms = max_over_ranks(elapsed_ms, device)
    max_serial_ms = max_over_ranks(serial_ms, device)

    # e2e: the same step through the public API from pinned host buffers
    e2e = run_e2e(args, host_calls, device, world)

    return dict(calls=calls, steps_per_step=steps_per_step, launches_per_step=launches_per_step,
                elapsed_ms=max_ms, serial_ms=max_serial_ms, streams=nstreams, per_call_ms=per_call_ms,
                per_group=per_group,
                group_ms_per_step=group_ms_total / args.steps, clocks=clocks, e2e=e2e,
                warmup=warm_done, status=status)


def run_e2e(args, host_calls, device, world):
    import torch
    import torch.distributed as dist

    import segmented_linear_recurrence_b200 as slr
    pinned = []
    h2d = d2h = 0
    tm, bf16 = time_major(args.workload), bf16_io(args.workload)
    for est, T, d in host_calls:
        ins = []
        for k, a in zip(ARG_ORDER[est], call_arrays(est, d, tm)):
            t = None if a is None else torch.from_numpy(a)
            if t is not None and bf16 and k in REAL_KEYS:
                t = t.to(torch.bfloat16)
            ins.append(None if t is None else t.pin_memory())
        h2d += sum(x.numel() * x.element_size() for x in ins if x is not None)
        shape = d["q"].shape[:2] if est == "retrace" else d[ARG_ORDER[est][0]].shape
        d2h += (2 if bf16 else 4) * int(np.prod(shape)) * len(OUT_KW[est])
        scal = {} if est == "episodic_prefix_sum" else dict(synthetic.SCALARS[est])
        pinned.append((f"rlscan_{est}{'_tm' if tm else ''}{'_bf16' if bf16 else ''}", ins, scal))

    def step():
        out = None
        for fn, ins, scal in pinned:
            out = getattr(slr, fn)(*ins, **scal)
        return out

    step()  # warm the caching allocators
    torch.cuda.synchronize()
    n = max(1, args.e2e_steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), device)
    return dict(ms_per_step=ms / n, steps=n, h2d=h2d, d2h=d2h)


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_pass(host_calls):
    import oracle
    steps = 0
    for est, T, d in host_calls:
        oracle.run(est, d, **synthetic.SCALARS[est])
        steps += d["q"].shape[0] * d["q"].shape[1] if est == "retrace" else int(np.prod(
            d[ARG_ORDER[est][0]].shape))
    return steps


def cpu_baseline(host_calls, seconds: float):
    """Times the oracle (single-threaded plain C loops) over whole passes of
    the workload until at least `seconds` of CPU work has run."""
    oracle_pass([host_calls[0]])  # build / load
    done_steps, passes = 0, 0
    t0 = time.perf_counter()
    while True:
        done_steps += oracle_pass(host_calls)
        passes += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    line = {"value": done_steps / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{passes} full pass(es) over the workload ({done_steps} env-steps, "
                      f"{dt:.1f} s, one thread, fp64)"}
    line.update(cpu_baseline_all_cores(host_calls, seconds / 2))
    return line


def cpu_baseline_all_cores(host_calls, seconds: float):
    """The same oracle on every host core: each call's rows split into one
    slice per thread (the C loops release the interpreter lock), whole passes
    until at least `seconds` have run.  Reported beside the one-thread value."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    workers = max(1, os.cpu_count() or 1)

    def sliced(d, lo, hi):
        return {k: (None if v is None else v[lo:hi]) for k, v in d.items()}

    def one_pass(pool):
        futs, steps = [], 0
        for est, T, d in host_calls:
            N = d["q"].shape[0] if est == "retrace" else d[ARG_ORDER[est][0]].shape[0]
            steps += N * T
            per = -(-N // workers)
            for lo in range(0, N, per):
                futs.append(pool.submit(oracle.run, est, sliced(d, lo, min(N, lo + per)), **synthetic.SCALARS[est]))
        for f in futs:
            f.result()
        return steps

    with ThreadPoolExecutor(max_workers=workers) as pool:
        one_pass(pool)  # warm
        done, passes = 0, 0
        t0 = time.perf_counter()
        while True:
            done += one_pass(pool)
            passes += 1
            if time.perf_counter() - t0 >= seconds:
                break
        dt = time.perf_counter() - t0
    return {"all_cores_value": done / dt, "all_cores": workers,
            "all_cores_sample": f"{passes} full pass(es), rows split over {workers} threads, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    host_calls = workload_calls(args.workload, 0)
    per_pass = oracle_pass([host_calls[0]])  # build / load
    for _ in range(max(args.warmup, 0)):
        oracle_pass(host_calls)
    t0 = time.perf_counter()
    steps = 0
    for _ in range(args.steps):
        steps += oracle_pass(host_calls)
    dt = time.perf_counter() - t0
    value = steps / dt
    cores = 1
    w = synthetic.WORKLOADS[args.workload]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "estimators": list(w["estimators"]), "N_envs": w["N"],
                   "T": list(w["Ts"]), "implementation": "fp64 sequential CPU oracle (oracle/)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} full pass(es) over the workload, one thread"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    del per_pass
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
def run_one(args):
    """`--one EST N T [A]`: `--steps` plain calls of one estimator on seeded
    inputs of the workload recipe (p_term 0.02, p_trunc 0.005 where the
    estimator takes truncation), for ncu captures of a single kernel.  EST
    with a `_tm` suffix runs the time-major entry point."""
    import torch
    import segmented_linear_recurrence_b200 as slr
    from segmented_linear_recurrence_b200 import build as slr_build
    slr_build.build()
    est, N, T = args.one[0], int(args.one[1]), int(args.one[2])
    tm = est.endswith("_tm")
    est = est[:-3] if tm else est
    A = int(args.one[3]) if len(args.one) > 3 else 18
    trunc = 0.0 if est in ("retrace", "elig_trace", "episodic_prefix_sum") else 0.005
    if est == "affine_scan":
        d = synthetic.make_affine_inputs(N, T, seed=5, p_reset=0.02)
    else:
        d = synthetic.make_inputs(est, N, T, seed=5, p_term=0.02, p_trunc=trunc, A=A, with_init=True)
    call = DeviceCall(est, T, d, torch.device("cuda", 0), tm)
    for _ in range(max(args.steps, 1)):
        call.launch()
    torch.cuda.synchronize()
    st = slr.rlscan_sync_status()
    print(json.dumps({"one": est + ("_tm" if tm else ""), "N": N, "T": T, "A": A, "calls": args.steps,
                      "status": st}))
    return 0 if st == 0 else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=tuple(synthetic.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--streams", type=int, default=4,
                    help="streams the step's independent estimators run on (1: one stream, in order)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work for the oracle baseline (0 disables it)")
    ap.add_argument("--one", nargs="+", metavar="EST N T [A]",
                    help="only run --steps plain calls of one estimator (for profiling)")
    args = ap.parse_args()

    if args.impl == "reference":
        return run_reference(args)
    if args.one:
        return run_one(args)

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_gpu(args, rank, world, local_rank)

    calls = res["calls"]
    ms_step = res["elapsed_ms"] / args.steps
    value = aggregate_rate(world, res["steps_per_step"], ms_step)
    peak, peak_kind = measured_peak()

    # per-estimator breakdown (group events, timed over K steps) and the
    # dominant kernel; per-T launch times from the per-launch-event graph
    per_est = {}
    for c, ms in zip(calls, res["per_call_ms"]):
        e = per_est.setdefault(c.est, {"bytes": 0, "steps": 0, "launches": 0, "by_T": {}})
        e["bytes"] += c.bytes
        e["steps"] += c.steps
        e["launches"] += 1
        gbs = c.bytes / (ms / 1000.0) / 1e9
        e["by_T"][str(c.T)] = {"us": round(ms * 1000.0, 2),
                               "gsteps_s": round(c.steps / (ms / 1000.0) / 1e9, 2),
                               "gbs": round(gbs, 1), "frac_of_measured": round(gbs / peak, 3),
                               "frac_of_8TBs": round(gbs / SPEC_HBM_GBS, 3)}
    for est, e in per_est.items():
        e["ms"] = res["per_group"][est]
    dom = max(per_est, key=lambda k: per_est[k]["ms"])
    de = per_est[dom]
    achieved = de["bytes"] / (de["ms"] / 1000.0) / 1e9
    tm = time_major(args.workload)
    dom_kernel = f"tm_scan_kernel<{dom}>" if tm else ("retrace_kernel" if dom == "retrace" else f"scan_kernel<{dom}>")
    if bf16_io(args.workload):
        dom_kernel = f"scan_kernel<{dom}, bf16 I/O>"
    traffic = load_traffic(args.workload, dom)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "kernel": dom_kernel, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_launch": int(de["bytes"] / de["launches"]),
                "avg_launch_us": round(1000.0 * de["ms"] / de["launches"], 2),
                "frac_of_8TBs_spec": round(achieved / SPEC_HBM_GBS, 4),
                "timing": "CUDA events around each estimator's launches inside the step graph, "
                          "averaged over the K timed steps"}

    e2e = res["e2e"]
    e2e_value = aggregate_rate(world, res["steps_per_step"], e2e["ms_per_step"])

    w = synthetic.WORKLOADS[args.workload]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": res["warmup"], "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 I/O, f32 arithmetic" if bf16_io(args.workload) else "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "estimators": list(w["estimators"]),
                   "N_envs_per_gpu": w["N"], "T": list(w["Ts"]), "p_term": w["p_term"],
                   "p_trunc": w["p_trunc"], "calls_per_step": len(calls),
                   "layout": "time-major [T, N]" if tm else "row-major [N, T]",
                   "l2": "inputs > L2: every call reads its own buffers; "
                         f"{sum(sum(x.numel() * x.element_size() for x in c.inputs if x is not None) for c in calls) / 1e9:.2f}"
                         " GB of distinct inputs per step",
                   "timing": "K replays of a CUDA graph holding one step's launches, CUDA events around the K",
                   "streams": res["streams"],
                   "parallelism": f"dp{world} (independent env shards, no collective)"},
        "roofline": roofline,
        "gpu_launches": int(res["launches_per_step"] * args.steps),
        "clocks": res["clocks"],
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(e2e["h2d"]),
                "d2h_bytes_per_step": int(e2e["d2h"]), "ms_per_step": e2e["ms_per_step"],
                "steps": e2e["steps"], "path": "public Python API on pinned host tensors"},
        "per_estimator": {k: {"gsteps_s": round(v["steps"] / (v["ms"] / 1000.0) / 1e9, 2),
                              "gbs": round(v["bytes"] / (v["ms"] / 1000.0) / 1e9, 1),
                              "frac_of_measured": round(v["bytes"] / (v["ms"] / 1000.0) / 1e9 / peak, 4),
                              "ms_per_step": round(v["ms"], 4),
                              "by_T_event_per_launch": v["by_T"]} for k, v in per_est.items()},
        "ms_per_step_with_group_events": res["group_ms_per_step"],
        "ms_per_step_one_stream": res["serial_ms"] / args.steps,
        "value_one_stream": aggregate_rate(world, res["steps_per_step"], res["serial_ms"] / args.steps),
        "device_status": res["status"],
    }
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        line["cpu_baseline"] = cpu_baseline(workload_calls(args.workload, 0), args.cpu_seconds)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
