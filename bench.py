"""Benchmark of the MoE layout -> dispatch -> combine step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 2]

One step = the whole token-choice hot path on one batch: the layout and the
bf16 compact dispatch (ep_layout_dispatch: ep_get_layout + ep_dispatch in one
call) and ep_combine (gate-weighted, fp32 accumulate, bf16 out), the expert
function between them being the identity.  Default workload: 4096 tokens x 7168 hidden, 256 experts in 8
logical ranks, top-8 (sigmoid router with bias), seeded synthetic inputs.

Timing: W untimed warm-up steps; then K steps, each preceded by a 256 MiB
memset that flushes the 126 MB L2 outside the timed events; CUDA events on
the launching stream around every step and every kernel; barrier + device
synchronize on both sides; the max over ranks.  value = algorithmic HBM bytes
of all steps on all ranks / max time (GB/s).  With N > 1 (torchrun) every rank
runs its own token batch (its own seed): the units are independent, there is
no collective on the data path, and the scaling is weak.
"""
from __future__ import annotations

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
sys.path.insert(0, ROOT)

METRIC = "dispatch+combine HBM GB/s and tokens/s at 4096×7168 top-8; % of HBM peak"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, choices=[2, 5])
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--e2e-chunks", type=int, default=8, help="token chunks of the pipelined end-to-end step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the per-op timings of the decode, expert-choice and skewed workloads")
    ap.add_argument("--other-reps", type=int, default=30)
    ap.add_argument("--print-digests", action="store_true", help="print kernel source digests and exit")
    ap.add_argument("--workloads", action="store_true",
                    help="time every op on all five workloads (one JSON line each) instead of the step")
    ap.add_argument("--only", type=int, default=0, choices=[0, 1, 2, 3, 4, 5],
                    help="with --workloads: just this workload")
    ap.add_argument("--quant", action="store_true",
                    help="with --workloads: also time every quantised dispatch format on the token-choice workloads")
    ap.add_argument("--ranks", action="store_true",
                    help="with --workloads: also time the per-rank (deduplicated) dispatch and combine, "
                         "and the same over peer memory with the ranks emulated on this GPU")
    ap.add_argument("--rounds", type=int, default=0,
                    help="with --workloads: also time the whole batch in rounds of this many tokens "
                         "(per-round layout, dispatch and combine; receive buffer of one round)")
    return ap.parse_args()


def algorithmic_bytes(cfg, n_valid):
    """HBM bytes the step must move, by kernel (each input read once, each
    output written once)."""
    T, H, K, R, E = cfg["T"], cfg["H"], cfg["K"], cfg["R"], cfg["E"]
    layout = T * K * 8 + T * K * 4 + T * R + E * 4 * 2 + 4 + R * 4
    dispatch = T * H * 2 + n_valid * H * 2 + T * K * 8 + T * K * 4 + E * 4
    combine = n_valid * H * 2 + T * H * 2 + T * K * 8 + T * K * 4 + T * K * 4 + E * 4
    return dict(layout=layout, dispatch=dispatch, combine=combine)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {"layout": "ep_layout.cu", "dispatch": "ep_dispatch.cu", "combine": "ep_combine.cu"}


def source_digest(kernel):
    """Digest of the sources a kernel is compiled from (its .cu file and the
    shared headers): a recorded ncu traffic figure is valid only for it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_ep_get_10_b200", "csrc")
    for name in sorted([KERNEL_SOURCES[kernel], "ep_device.cuh", "ep_internal.h"]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(ROOT, "include", "ep.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = source_digest(kernel)
    for line in open(path):
        fields = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if fields.get("kernel") == kernel and fields.get("source_sha") == want:
            try:
                return int(fields["dram_bytes_per_launch"])
            except (KeyError, ValueError):
                return None
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, uuid=None):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(index)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = self._reasons_fn(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0,
                    "source": "nvml unavailable" if self._nv is None else "nvml"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (n_gpus, world))
    return world, rank, local


def rank_seed(workload, rank):
    """Seed of rank `rank`'s token batch: the workload seed for rank 0, then
    one independent stream per rank (replicas on disjoint data)."""
    from combine_ep_get_10_b200 import workloads as W

    return W.CONFIGS[workload]["seed"] + 1000 * rank


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (all ranks must call it)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def host_cores():
    """Cores of this host (the oracle itself runs on one thread): what the OS
    reports and what this process may use."""
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = None
    return {"cpu_count": os.cpu_count(), "usable": usable}


def cpu_oracle_run(cfg_id, seed, n_tokens, reps_budget_s, min_reps=1):
    """Time the CPU oracle (single thread) on the first n_tokens tokens of the
    workload: layout + dispatch + combine, as a bounded sample."""
    import oracle
    from combine_ep_get_10_b200 import workloads as W

    inp = W.make_inputs(cfg_id, seed=seed)
    cfg = inp["cfg"]
    x = np.ascontiguousarray(inp["x"][:n_tokens])
    idx = np.ascontiguousarray(inp["topk_idx"][:n_tokens])
    w = np.ascontiguousarray(inp["topk_weights"][:n_tokens])
    sub = dict(cfg, T=n_tokens)
    n_valid = int((idx >= 0).sum())
    times = []
    t_end = time.perf_counter() + reps_budget_s
    while len(times) < min_reps or time.perf_counter() < t_end:
        t0 = time.perf_counter()
        L = oracle.tc_layout(idx, cfg["E"], cfg["R"])
        D = oracle.tc_dispatch(x, idx, cfg["E"], L)
        oracle.tc_combine(D["recv"], idx, cfg["E"], L, w, out_dtype=oracle.BF16)
        times.append(time.perf_counter() - t0)
    b = sum(algorithmic_bytes(sub, n_valid).values())
    return times, b


def run_reference(args):
    """The CPU oracle as the reference arm: every step is a bounded sample
    (the first 256 tokens of the workload), single-threaded on the host."""
    world, rank, _ = dist_setup(args.gpus)
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    from combine_ep_get_10_b200 import workloads as W

    cfg = W.CONFIGS[args.workload]
    n_tok = 256
    inp = W.make_inputs(args.workload)
    x = np.ascontiguousarray(inp["x"][:n_tok])
    idx = np.ascontiguousarray(inp["topk_idx"][:n_tok])
    w = np.ascontiguousarray(inp["topk_weights"][:n_tok])
    n_valid = int((idx >= 0).sum())
    bytes_step = sum(algorithmic_bytes(dict(cfg, T=n_tok), n_valid).values())

    def step():
        L = oracle.tc_layout(idx, cfg["E"], cfg["R"])
        D = oracle.tc_dispatch(x, idx, cfg["E"], L)
        oracle.tc_combine(D["recv"], idx, cfg["E"], L, w, out_dtype=oracle.BF16)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = bytes_step * args.steps / dt / 1e9
    sample = "first %d of %d tokens of workload %s per step" % (n_tok, cfg["T"], cfg["name"])
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": {"workload": cfg["name"], "sample_tokens": n_tok},
            "tokens_per_s": n_tok * args.steps / dt,
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                             "host_cores": host_cores()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    from combine_ep_get_10_b200 import binding as B
    from combine_ep_get_10_b200 import build as build_mod
    from combine_ep_get_10_b200 import workloads as W

    if not os.path.exists(build_mod.LIB) and rank == 0:
        build_mod.build()
    if world > 1:
        dist.barrier()
    B.lib()

    seed = rank_seed(args.workload, rank)
    inp = W.make_inputs(args.workload, seed=seed)
    cfg = inp["cfg"]
    T, H, K, E, R = cfg["T"], cfg["H"], cfg["K"], cfg["E"], cfg["R"]
    n_valid = int((inp["topk_idx"] >= 0).sum())
    nbytes = algorithmic_bytes(cfg, n_valid)
    step_bytes = sum(nbytes.values())

    dev = torch.device("cuda", local)
    x_h = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx_h = torch.from_numpy(inp["topk_idx"]).pin_memory()
    w_h = torch.from_numpy(inp["topk_weights"]).pin_memory()
    x = x_h.to(dev)
    idx = idx_h.to(dev)
    w = w_h.to(dev)
    routing = B.Routing.topk(idx, E, R)
    lay = B.Layout(routing, device=dev)
    recv = torch.empty((T * K, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        # layout + dispatch in one call (the dispatch's row loads overlap the
        # layout kernel), then the combine
        B.ep_layout_dispatch(x, routing, lay, recv, num_recv_rows=T * K, stream=stream)
        B.ep_combine(recv, routing, lay, w, out, num_y_rows=T * K, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if B.ep_get_device_error(lay) != 0:
        raise RuntimeError("device error flagged during warm-up")

    K_steps = args.steps
    es = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    uuid = ("GPU-" + str(props.uuid)) if getattr(props, "uuid", None) is not None else None
    with ClockSampler(local, uuid) as clocks:
        # the timed steps: events only around each step (an event recorded
        # between two kernels delays the second one's start)
        for i in range(K_steps):
            flush.zero_()
            es[i][0].record(stream)
            step()
            es[i][1].record(stream)
        torch.cuda.synchronize(dev)
        # the per-kernel breakdown: K more steps with events between the kernels
        for i in range(K_steps):
            flush.zero_()
            e0, e1, e2, e3 = ev[i]
            e0.record(stream)
            B.ep_get_layout(routing, lay, stream=stream)
            e1.record(stream)
            B.ep_dispatch(x, routing, lay, recv, num_recv_rows=T * K, stream=stream)
            e2.record(stream)
            B.ep_combine(recv, routing, lay, w, out, num_y_rows=T * K, stream=stream)
            e3.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t_layout = [a[0].elapsed_time(a[1]) for a in ev]
    t_disp = [a[1].elapsed_time(a[2]) for a in ev]
    t_comb = [a[2].elapsed_time(a[3]) for a in ev]
    t_step_split = [a[0].elapsed_time(a[3]) for a in ev]
    t_step = [a[0].elapsed_time(a[1]) for a in es]
    total_ms = max_over_ranks(float(sum(t_step)), world, dev)
    if B.ep_get_device_error(lay) != 0:
        raise RuntimeError("device error flagged during the timed steps")

    # end to end through the public API with host buffers: pinned H2D of the
    # step's inputs, the three calls, D2H of the combined output.  The token
    # batch is cut into chunks so that the H2D of chunk c+1 and the D2H of
    # chunk c-1 (two copy streams) overlap the dispatch + combine of chunk c.
    out_h = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(1, min(args.e2e_steps, K_steps))
    h2d = x_h.numel() * 2 + idx_h.numel() * 8 + w_h.numel() * 4
    d2h = out_h.numel() * 2
    n_chunks = max(1, min(args.e2e_chunks, T))
    bounds = [T * c // n_chunks for c in range(n_chunks + 1)]
    s_in = torch.cuda.Stream(dev)
    views = [(routing.tokens(a, b), B.layout_tokens(lay, routing, a, b), a, b) for a, b in zip(bounds[:-1], bounds[1:])]

    def e2e_step(ev0, ev1):
        ev0.record(stream)
        s_in.wait_event(ev0)
        with torch.cuda.stream(s_in):
            idx.copy_(idx_h, non_blocking=True)
            w.copy_(w_h, non_blocking=True)
            ev_meta = torch.cuda.Event()
            ev_meta.record(s_in)
            ev_x = []
            for r_c, v_c, a, b in views:
                x[a:b].copy_(x_h[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(s_in)
                ev_x.append(e)
        stream.wait_event(ev_meta)
        B.ep_get_layout(routing, lay, stream=stream)
        for (r_c, v_c, a, b), e in zip(views, ev_x):
            stream.wait_event(e)
            B.ep_dispatch(x[a:b], r_c, v_c, recv, num_recv_rows=T * K, stream=stream)
            # the combine writes the chunk's result straight into pinned host
            # memory (mapped under unified addressing): the device->host
            # transfer is the kernel's own stores over PCIe, overlapping the
            # host->device copies of the later chunks
            B.ep_combine(recv, r_c, v_c, w[a:b], out_h[a:b], num_y_rows=T * K, stream=stream)
        ev1.record(stream)

    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps + 2)]
    for i in range(2):  # untimed warm-up of the pipelined path
        flush.zero_()
        e2e_step(*ee[i])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(2, e2e_steps + 2):
        flush.zero_()
        e2e_step(*ee[i])
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(float(sum(a.elapsed_time(b) for a, b in ee[2:])), world, dev)
    if world > 1:
        dist.barrier()
    if B.ep_get_device_error(lay) != 0:
        raise RuntimeError("device error flagged during the end-to-end steps")

    # the other workloads' ops, timed in this process with clocks sampled
    # (one GPU only: under torchrun the other ranks would wait at the final
    # barrier meanwhile)
    other, other_clocks = None, None
    if world == 1 and not args.no_other_workloads:
        with ClockSampler(local, uuid) as clocks2:
            other = time_other_workloads(dev, flush, args.other_reps)
        other_clocks = clocks2.summary()

    if rank == 0:
        peak, peak_kind = measured_peak()
        mean = lambda a: float(sum(a) / len(a))  # noqa: E731
        k_ms = {"layout": mean(t_layout), "dispatch": mean(t_disp), "combine": mean(t_comb)}
        dominant = max(("dispatch", "combine"), key=lambda k: k_ms[k])
        achieved = nbytes[dominant] / (k_ms[dominant] * 1e-3) / 1e9
        traffic = recorded_traffic(dominant)
        value = step_bytes * K_steps * world / (total_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K_steps,
            "warmup": max(3, args.warmup), "ms_per_step": total_ms / K_steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded numpy PCG64 per rank; no dataset)",
            "config": {"workload": cfg["name"], "num_tokens": T, "hidden": H, "num_topk": K, "num_experts": E,
                       "logical_ranks": R, "valid_pairs": n_valid, "dispatch": "bf16 compact",
                       "combine": "bf16 out, fp32 accumulate", "l2": "flushed: 256 MiB memset before every step",
                       "parallelism": "replicas, one token batch per GPU" if world > 1 else "single GPU"},
            "tokens_per_s": T * K_steps * world / (total_ms * 1e-3),
            "kernels_us": {k: v * 1e3 for k, v in k_ms.items()},
            "kernels_timing": "a second pass of the same %d steps as separate ep_get_layout / ep_dispatch / ep_combine "
                              "calls with CUDA events between the kernels (those steps take %.1f us each; the timed "
                              "steps, events only around each step, %.1f us)"
                              % (K_steps, mean(t_step_split) * 1e3, total_ms / K_steps * 1e3),
            "kernels_gbs": {k: nbytes[k] / (k_ms[k] * 1e-3) / 1e9 for k in k_ms},
            "algorithmic_bytes_per_step": nbytes,
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind, "traffic": traffic,
                         "frac_of_nominal_8000_gbs": achieved / 8000.0,
                         "step_frac": value / peak},
            "gpu_launches": 3 * K_steps,
            "e2e": {"value": step_bytes * e2e_steps * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "tokens_per_s": T * e2e_steps * world / (e2e_ms * 1e-3), "steps": e2e_steps,
                    "token_chunks": n_chunks, "copies": "pinned host: H2D chunks on a copy stream overlapping compute; the combine "
                                                 "writes the result into pinned host memory (zero-copy D2H)",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "clocks": clocks.summary(),
        }
        if other is not None:
            line["other_workloads"] = {"per_op": other, "reps": args.other_reps,
                                       "timing": "CUDA events around each op alone, L2 flushed (256 MiB memset) "
                                                 "before each repetition, median; frac against the same peak",
                                       "clocks": other_clocks}
        if world == 1 and not args.no_cpu_baseline:
            n_tok = 1024
            times, b = cpu_oracle_run(args.workload, seed, n_tok, reps_budget_s=10.0)
            med = statistics.median(times)
            line["cpu_baseline"] = {"value": b / med / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                    "host_cores": host_cores(),
                                    "sample": "first %d of %d tokens, layout+dispatch+combine, median of %d reps"
                                              % (n_tok, T, len(times)),
                                    "tokens_per_s": n_tok / med}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_other_workloads(dev, flush, reps):
    """Per-op event timings of the decode (3), expert-choice (4) and skewed
    (5) workloads, and of the prefill workload's quantised, per-rank and
    peer-path rows, each op alone after an L2 flush, median of `reps`;
    returned as {workload: {op: {"us", "gbs", "frac", "bytes"}}} for the
    bench line."""
    import torch

    from combine_ep_get_10_b200 import binding as B
    from combine_ep_get_10_b200 import workloads as W

    peak, _ = measured_peak()
    spread = {}  # min, p90 and mean of the last timeit, for the record that reports it

    def timeit(fn):
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(dev)
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        ts.sort()
        spread.update(us_min=ts[0], us_p90=ts[min(len(ts) - 1, (9 * len(ts)) // 10)], us_mean=sum(ts) / len(ts))
        return statistics.median(ts)

    def rec(us, nbytes):
        return {"us": round(us, 2), **{k: round(v, 2) for k, v in spread.items()}, "bytes": int(nbytes),
                "gbs": round(nbytes / us / 1e3, 1), "frac": round(nbytes / us / 1e3 / peak, 3)}

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    res = {}
    for wl in (3, 4, 5):
        inp = W.make_inputs(wl)
        cfg = inp["cfg"]
        T, H, E, R = cfg["T"], cfg["H"], cfg["E"], cfg["R"]
        x = bf(inp["x"])
        ops = {}
        if cfg["routing"] == "topk":
            K = cfg["K"]
            n_valid = int((inp["topk_idx"] >= 0).sum())
            idx = torch.from_numpy(inp["topk_idx"]).to(dev)
            w = torch.from_numpy(inp["topk_weights"]).to(dev)
            rt = B.Routing.topk(idx, E, R)
            lay = B.Layout(rt, device=dev)
            ops["layout"] = rec(timeit(lambda: B.ep_get_layout(rt, lay)), T * K * 12 + T * R + E * 8 + R * 4)
            mode, mt = cfg["mode"], cfg["max_tokens"]
            rows = E * mt if mode == W.PADDED else T * K
            meta = T * K * 12 + E * 4
            y = torch.zeros((rows, H), dtype=torch.bfloat16, device=dev)
            if cfg["dispatch_dtype"] == W.FP8_E4M3:
                q = torch.empty((rows, H), dtype=torch.uint8, device=dev)
                sc = torch.empty((rows, H // 128), dtype=torch.float32, device=dev)
                ops["dispatch_fp8"] = rec(timeit(lambda: B.ep_dispatch(x, rt, lay, q, mode=mode, max_tokens_per_expert=mt,
                                                                      recv_scales=sc)),
                                          T * H * 2 + n_valid * (H + H // 128 * 4) + meta)
                ops["low_latency_layout_dispatch_fp8"] = rec(
                    timeit(lambda: B.ep_dispatch_low_latency(x, rt, lay, q, max_tokens_per_expert=mt, recv_scales=sc)),
                    T * K * 12 + T * R + E * 8 + R * 4 + T * H * 2 + n_valid * (H + H // 128 * 4))
                del q, sc
            else:
                ops["dispatch"] = rec(timeit(lambda: B.ep_dispatch(x, rt, lay, y, mode=mode, max_tokens_per_expert=mt)),
                                      T * H * 2 + n_valid * H * 2 + meta)
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            ops["combine"] = rec(timeit(lambda: B.ep_combine(y, rt, lay, w, out, mode=mode, max_tokens_per_expert=mt)),
                                 n_valid * H * 2 + T * H * 2 + T * K * 16 + E * 4)
        else:
            C = cfg["C"]
            ti_np = inp["token_indices"]
            S = E * C
            uniq = len(np.unique(ti_np[ti_np >= 0]))
            ti = torch.from_numpy(ti_np).to(dev)
            ew = torch.from_numpy(inp["expert_weights"]).to(dev)
            rt = B.Routing.expert_choice(ti, T, R)
            lay = B.Layout(rt, device=dev)
            ops["ec_layout"] = rec(timeit(lambda: B.ep_get_layout(rt, lay)), S * 4 + (T + 1) * 4 + S * 4 + T * R + E * 4 + R * 4)
            y = torch.empty((S, H), dtype=torch.bfloat16, device=dev)
            ops["ec_dispatch"] = rec(timeit(lambda: B.ep_dispatch_expert_choice(x, rt, lay, y)), uniq * H * 2 + S * H * 2 + S * 4)
            ops["ec_layout_dispatch"] = rec(timeit(lambda: B.ep_layout_dispatch_expert_choice(x, rt, lay, y)),
                                            S * 4 + (T + 1) * 4 + S * 4 + T * R + E * 4 + R * 4
                                            + uniq * H * 2 + S * H * 2 + S * 4)
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            ops["ec_combine"] = rec(timeit(lambda: B.ep_combine_expert_choice(y, rt, lay, ew, out)),
                                    S * H * 2 + T * H * 2 + S * 8 + (T + 1) * 4)
        if B.ep_get_device_error(lay) != 0:
            raise RuntimeError("device error flagged on workload %d" % wl)
        res[cfg["name"]] = ops
        del x, y, out, lay
        torch.cuda.empty_cache()
    res["prefill-topk-4096x7168-top8 (quantised, per-rank and peer-path rows)"] = time_prefill_rows(
        dev, timeit, rec, bf)
    torch.cuda.empty_cache()
    return res


def time_prefill_rows(dev, timeit, rec, bf):
    """The prefill workload's other rows: every quantised dispatch format
    (compact), the per-rank (deduplicated) dispatch and combine, and the
    same over peer memory with the ranks emulated on this GPU."""
    import torch

    from combine_ep_get_10_b200 import binding as B
    from combine_ep_get_10_b200 import workloads as W

    inp = W.make_inputs(2)
    cfg = inp["cfg"]
    T, H, E, R, K = cfg["T"], cfg["H"], cfg["E"], cfg["R"], cfg["K"]
    x = bf(inp["x"])
    n_valid = int((inp["topk_idx"] >= 0).sum())
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    w = torch.from_numpy(inp["topk_weights"]).to(dev)
    rt = B.Routing.topk(idx, E, R)
    lay = B.Layout(rt, device=dev)
    B.ep_get_layout(rt, lay)
    ops = {}
    meta = T * K * 12 + E * 4
    for name, dt, code_b, scale_b in QUANT_FORMATS:
        cb, sb = code_b(H), scale_b(H)
        q = torch.empty((n_valid, cb), dtype=torch.uint8, device=dev)
        sc = torch.empty((n_valid, sb), dtype=torch.uint8, device=dev)
        ops["dispatch_" + name] = rec(timeit(lambda: B.ep_dispatch(x, rt, lay, q, recv_scales=sc, out_dtype=dt)),
                                      T * H * 2 + n_valid * (cb + sb) + meta)
        del q, sc
    rl = B.RankLayout(rt, device=dev)
    ops["rank_layout"] = rec(timeit(lambda: B.ep_get_rank_layout(rt, lay, rl)),
                             T * R + R * 4 + (R + 1) * 4 + T * R * 4)
    n_rank = int(rl.rank_offsets[-1].item())
    rrecv = torch.empty((n_rank, H), dtype=torch.bfloat16, device=dev)
    ridx = torch.empty((n_rank, K), dtype=torch.int64, device=dev)
    rwt = torch.empty((n_rank, K), dtype=torch.float32, device=dev)
    ops["dispatch_ranks"] = rec(timeit(lambda: B.ep_dispatch_ranks(x, rt, lay, rl, rrecv, topk_weights=w,
                                                                   recv_topk_idx=ridx, recv_topk_weights=rwt)),
                                T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + T * R * 4 + T * K * 12)
    ops["layout_dispatch_ranks"] = rec(
        timeit(lambda: B.ep_layout_dispatch_ranks(x, rt, lay, rl, rrecv, topk_weights=w, recv_topk_idx=ridx,
                                                  recv_topk_weights=rwt)),
        T * K * 12 + T * R + E * 8 + R * 4 + T * R + R * 4 + (R + 1) * 4 + T * R * 4
        + T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + T * R * 4 + T * K * 12)
    rout = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ops["combine_ranks"] = rec(timeit(lambda: B.ep_combine_ranks(rrecv, rt, lay, rl, rout)),
                               n_rank * H * 2 + T * H * 2 + T * R * 4)
    del rrecv, ridx, rwt, rout
    time_peer_path(cfg, x, w, rt, lay, rl, n_rank, dev, timeit,
                   lambda cfg_, op, us, nbytes, tokens: ops.__setitem__(op, rec(us, nbytes)))
    if B.ep_get_device_error(lay) != 0:
        raise RuntimeError("device error flagged on the prefill rows")
    return ops


# quantised dispatch formats: (name, dtype code, code bytes per row, scale bytes per row)
QUANT_FORMATS = [
    ("fp8_g128", 2, lambda H: H, lambda H: H // 128 * 4),
    ("int8_per_token", 3, lambda H: H, lambda H: 4),
    ("fp8_per_token", 4, lambda H: H, lambda H: 4),
    ("mxfp8_e4m3", 5, lambda H: H, lambda H: H // 32),
    ("mxfp8_e5m2", 6, lambda H: H, lambda H: H // 32),
    ("mxfp4_e2m1", 7, lambda H: H // 2, lambda H: H // 32),
]


def time_peer_path(cfg, x, w, rt, lay, rl, n_rank, dev, timeit, emit):
    """The per-rank path over peer memory, its R ranks emulated on this GPU:
    this process is rank R/2 of R ranks that all hold this routing (so every
    row of the counts matrix is this rank's num_tokens_per_rank), and each
    rank's receive, entry, source and partial-row buffers are separate
    allocations here.  The dispatch stores this rank's (token, rank) rows
    into the R ranks' buffers at their offsets behind ranks 0 .. R/2-1, and
    the combine reads them back from there: the same bytes as
    dispatch_ranks / combine_ranks, over local HBM instead of NVLink."""
    import torch

    from combine_ep_get_10_b200 import binding as B

    T, H, K, R = cfg["T"], cfg["H"], cfg["K"], cfg["R"]
    me = R // 2
    counts = lay.num_tokens_per_rank.to(torch.int32)
    capacity = (me + 1) * int(counts.max().item())
    bufs = dict(recv_x=[torch.empty((capacity, H), dtype=torch.bfloat16, device=dev) for _ in range(R)],
                y=[torch.randn((capacity, H), device=dev).to(torch.bfloat16) for _ in range(R)],
                idx=[torch.empty((capacity, K), dtype=torch.int64, device=dev) for _ in range(R)],
                w=[torch.empty((capacity, K), dtype=torch.float32, device=dev) for _ in range(R)],
                src=[torch.empty((capacity,), dtype=torch.int32, device=dev) for _ in range(R)],
                counts=[counts.repeat(R, 1).contiguous() for _ in range(R)])
    tab = {k: torch.tensor([t.data_ptr() for t in v], dtype=torch.int64, device=dev) for k, v in bufs.items()}
    peers = B.Peers(me, capacity, tab["recv_x"], tab["y"], tab["counts"], recv_topk_idx=tab["idx"],
                    recv_topk_weights=tab["w"], recv_src=tab["src"])
    emit(cfg, "dispatch_peers_emulated",
         timeit(lambda: B.ep_dispatch_peers(x, rt, lay, rl, peers, topk_weights=w)),
         T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + n_rank * 4 + T * R * 4 + T * K * 12, T)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    emit(cfg, "combine_peers_emulated", timeit(lambda: B.ep_combine_peers(rt, lay, rl, peers, out)),
         n_rank * H * 2 + T * H * 2 + T * R * 4, T)
    del bufs, tab, peers, out


def run_workload_table(args):
    """Per-op timings on every workload (layout, dispatch, combine; expert
    choice for workload 4): one JSON line per (workload, op), L2 flushed
    before every repetition, median of --steps repetitions."""
    import torch

    from combine_ep_get_10_b200 import binding as B
    from combine_ep_get_10_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peak, peak_kind = measured_peak()
    reps = max(10, min(args.steps, 200))
    spread = {}  # min, p90 and mean of the last timeit, for the line that reports it

    def timeit(fn):
        ts = []
        for i in range(reps + 3):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        ts.sort()
        spread.update(us_min=ts[0], us_p90=ts[min(len(ts) - 1, (9 * len(ts)) // 10)], us_mean=sum(ts) / len(ts))
        return ts[len(ts) // 2]

    def emit(cfg, op, us, nbytes, tokens):
        print(json.dumps({"workload": cfg["name"], "op": op, "us": round(us, 2),
                          **{k: round(v, 2) for k, v in spread.items()}, "bytes": int(nbytes),
                          "gbs": round(nbytes / us / 1e3, 1), "frac_of_peak": round(nbytes / us / 1e3 / peak, 3),
                          "peak_gbs": peak, "peak_source": peak_kind, "tokens_per_s": round(tokens / us * 1e6),
                          "reps": reps, "l2": "flushed"}), flush=True)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    for wl in ([args.only] if args.only else (1, 2, 3, 4, 5)):
        inp = W.make_inputs(wl)
        cfg = inp["cfg"]
        T, H, E, R = cfg["T"], cfg["H"], cfg["E"], cfg["R"]
        x = bf(inp["x"])
        if cfg["routing"] == "topk":
            K = cfg["K"]
            idx_np = inp["topk_idx"]
            n_valid = int((idx_np >= 0).sum())
            idx = torch.from_numpy(idx_np).to(dev)
            w = torch.from_numpy(inp["topk_weights"]).to(dev)
            rt = B.Routing.topk(idx, E, R)
            lay = B.Layout(rt, device=dev)
            emit(cfg, "layout", timeit(lambda: B.ep_get_layout(rt, lay)),
                 T * K * 12 + T * R + E * 8 + R * 4, T)
            mode, mt = cfg["mode"], cfg["max_tokens"]
            rows = E * mt if mode == W.PADDED else T * K
            meta = T * K * 12 + E * 4
            if cfg["dispatch_dtype"] == W.FP8_E4M3:
                recv = torch.empty((rows, H), dtype=torch.uint8, device=dev)
                sc = torch.empty((rows, H // 128), dtype=torch.float32, device=dev)
                emit(cfg, "dispatch_fp8", timeit(lambda: B.ep_dispatch(x, rt, lay, recv, mode=mode,
                                                                       max_tokens_per_expert=mt, recv_scales=sc)),
                     T * H * 2 + n_valid * (H + H // 128 * 4) + meta, T)
                if mode == W.PADDED:  # layout + padded FP8 dispatch in one call
                    ll_bytes = T * K * 12 + T * R + E * 8 + R * 4 + T * H * 2 + n_valid * (H + H // 128 * 4)
                    emit(cfg, "low_latency_layout_dispatch_fp8",
                         timeit(lambda: B.ep_dispatch_low_latency(x, rt, lay, recv, max_tokens_per_expert=mt,
                                                                  recv_scales=sc)), ll_bytes, T)
                    # the decode step (fused dispatch + padded combine) replayed from a CUDA graph
                    yy = torch.zeros((rows, H), dtype=torch.bfloat16, device=dev)
                    oo = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
                    gs = torch.cuda.Stream(dev)

                    def decode_step():
                        B.ep_dispatch_low_latency(x, rt, lay, recv, max_tokens_per_expert=mt, recv_scales=sc,
                                                  stream=gs)
                        B.ep_combine(yy, rt, lay, w, oo, mode=mode, max_tokens_per_expert=mt, stream=gs)

                    gs.wait_stream(torch.cuda.current_stream(dev))
                    decode_step()
                    torch.cuda.synchronize(dev)
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph, stream=gs):
                        decode_step()
                    step_bytes_ll = ll_bytes + n_valid * H * 2 + T * H * 2 + T * K * 16 + E * 4
                    emit(cfg, "decode_step_eager (fused dispatch + combine)",
                         timeit(lambda: (B.ep_dispatch_low_latency(x, rt, lay, recv, max_tokens_per_expert=mt,
                                                                   recv_scales=sc),
                                         B.ep_combine(yy, rt, lay, w, oo, mode=mode, max_tokens_per_expert=mt))),
                         step_bytes_ll, T)
                    emit(cfg, "decode_step_cuda_graph (fused dispatch + combine)", timeit(graph.replay),
                         step_bytes_ll, T)
                    del graph
                y = torch.zeros((rows, H), dtype=torch.bfloat16, device=dev)
            else:
                recv = torch.empty((rows, H), dtype=torch.bfloat16, device=dev)
                emit(cfg, "dispatch", timeit(lambda: B.ep_dispatch(x, rt, lay, recv, mode=mode,
                                                                   max_tokens_per_expert=mt)),
                     T * H * 2 + n_valid * H * 2 + meta, T)
                lb = T * K * 12 + T * R + E * 8 + R * 4
                emit(cfg, "layout + dispatch (two calls)",
                     timeit(lambda: (B.ep_get_layout(rt, lay),
                                     B.ep_dispatch(x, rt, lay, recv, mode=mode, max_tokens_per_expert=mt))),
                     lb + T * H * 2 + n_valid * H * 2 + meta, T)
                emit(cfg, "layout + dispatch (one call, ep_layout_dispatch)",
                     timeit(lambda: B.ep_layout_dispatch(x, rt, lay, recv, mode=mode, max_tokens_per_expert=mt)),
                     lb + T * H * 2 + n_valid * H * 2 + meta, T)
                y = recv
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            emit(cfg, "combine", timeit(lambda: B.ep_combine(y, rt, lay, w, out, mode=mode,
                                                             max_tokens_per_expert=mt)),
                 n_valid * H * 2 + T * H * 2 + T * K * 16 + E * 4, T)
            if args.rounds and mode == W.COMPACT and args.rounds < T:
                P = args.rounds
                rnd = [(t0, min(T, t0 + P)) for t0 in range(0, T, P)]
                rr = [rt.tokens(t0, t1) for t0, t1 in rnd]
                rl = [B.Layout(r, device=dev) for r in rr]
                rbuf = torch.empty((P * K, H), dtype=torch.bfloat16, device=dev)
                rout = torch.empty((T, H), dtype=torch.bfloat16, device=dev)

                def all_rounds():
                    for (t0, t1), r, l in zip(rnd, rr, rl):
                        B.ep_get_layout(r, l)
                        B.ep_dispatch(x[t0:t1], r, l, rbuf, num_recv_rows=P * K)
                        B.ep_combine(rbuf, r, l, w[t0:t1], rout[t0:t1], num_y_rows=P * K)

                us = timeit(all_rounds)
                nb = (T * K * 12 + T * R + (E * 8 + R * 4) * len(rnd)  # layouts
                      + T * H * 2 + n_valid * H * 2 + T * K * 12 + E * 4 * len(rnd)  # dispatches
                      + n_valid * H * 2 + T * H * 2 + T * K * 16)  # combines
                emit(cfg, "rounds_%dx%d_layout_dispatch_combine" % (len(rnd), P), us, nb, T)
                del rbuf, rout
            if args.ranks and mode == W.COMPACT:
                rl = B.RankLayout(rt, device=dev)
                emit(cfg, "rank_layout", timeit(lambda: B.ep_get_rank_layout(rt, lay, rl)),
                     T * R + R * 4 + (R + 1) * 4 + T * R * 4, T)
                B.ep_get_rank_layout(rt, lay, rl)
                n_rank = int(rl.rank_offsets[-1].item())
                rrecv = torch.empty((n_rank, H), dtype=torch.bfloat16, device=dev)
                ridx = torch.empty((n_rank, K), dtype=torch.int64, device=dev)
                rwt = torch.empty((n_rank, K), dtype=torch.float32, device=dev)
                emit(cfg, "dispatch_ranks",
                     timeit(lambda: B.ep_dispatch_ranks(x, rt, lay, rl, rrecv, topk_weights=w, recv_topk_idx=ridx,
                                                        recv_topk_weights=rwt)),
                     T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + T * R * 4 + T * K * 12, T)
                emit(cfg, "layout + rank layout + dispatch_ranks (three calls)",
                     timeit(lambda: (B.ep_get_layout(rt, lay), B.ep_get_rank_layout(rt, lay, rl),
                                     B.ep_dispatch_ranks(x, rt, lay, rl, rrecv, topk_weights=w, recv_topk_idx=ridx,
                                                         recv_topk_weights=rwt))),
                     T * K * 12 + T * R + E * 8 + R * 4 + T * R + R * 4 + (R + 1) * 4 + T * R * 4
                     + T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + T * R * 4 + T * K * 12, T)
                emit(cfg, "layout_dispatch_ranks (one call: layout, rank layout, dispatch)",
                     timeit(lambda: B.ep_layout_dispatch_ranks(x, rt, lay, rl, rrecv, topk_weights=w,
                                                               recv_topk_idx=ridx, recv_topk_weights=rwt)),
                     T * K * 12 + T * R + E * 8 + R * 4 + T * R + R * 4 + (R + 1) * 4 + T * R * 4
                     + T * H * 2 + n_rank * H * 2 + n_rank * K * 12 + T * R * 4 + T * K * 12, T)
                rout = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
                emit(cfg, "combine_ranks", timeit(lambda: B.ep_combine_ranks(rrecv, rt, lay, rl, rout)),
                     n_rank * H * 2 + T * H * 2 + T * R * 4, T)
                print(json.dumps({"workload": cfg["name"], "rank_rows": n_rank, "expert_rows": n_valid,
                                  "rows_saved": round(1 - n_rank / max(n_valid, 1), 3)}), flush=True)
                del rrecv, ridx, rwt, rout
                time_peer_path(cfg, x, w, rt, lay, rl, n_rank, dev, timeit, emit)
            if args.quant:
                del recv
                for name, dt, code_b, scale_b in QUANT_FORMATS:
                    cb, sb = code_b(H), scale_b(H)
                    qrecv = torch.empty((rows, cb), dtype=torch.uint8, device=dev)
                    qsc = torch.empty((rows, sb), dtype=torch.uint8, device=dev)
                    emit(cfg, "dispatch_" + name,
                         timeit(lambda: B.ep_dispatch(x, rt, lay, qrecv, mode=mode, max_tokens_per_expert=mt,
                                                      recv_scales=qsc, out_dtype=dt)),
                         T * H * 2 + n_valid * (cb + sb) + meta, T)
                    del qrecv, qsc
        else:
            C = cfg["C"]
            ti_np = inp["token_indices"]
            S = E * C
            uniq = len(np.unique(ti_np[ti_np >= 0]))
            ti = torch.from_numpy(ti_np).to(dev)
            ew = torch.from_numpy(inp["expert_weights"]).to(dev)
            rt = B.Routing.expert_choice(ti, T, R)
            lay = B.Layout(rt, device=dev)
            emit(cfg, "ec_layout", timeit(lambda: B.ep_get_layout(rt, lay)),
                 S * 4 + (T + 1) * 4 + S * 4 + T * R + E * 4 + R * 4, T)
            recv = torch.empty((S, H), dtype=torch.bfloat16, device=dev)
            emit(cfg, "ec_dispatch", timeit(lambda: B.ep_dispatch_expert_choice(x, rt, lay, recv)),
                 uniq * H * 2 + S * H * 2 + S * 4, T)
            emit(cfg, "ec_layout + ec_dispatch (two calls)",
                 timeit(lambda: (B.ep_get_layout(rt, lay), B.ep_dispatch_expert_choice(x, rt, lay, recv))),
                 S * 4 + (T + 1) * 4 + S * 4 + T * R + E * 4 + R * 4 + uniq * H * 2 + S * H * 2 + S * 4, T)
            emit(cfg, "ec_layout_dispatch (one call)", timeit(lambda: B.ep_layout_dispatch_expert_choice(x, rt, lay, recv)),
                 S * 4 + (T + 1) * 4 + S * 4 + T * R + E * 4 + R * 4 + uniq * H * 2 + S * H * 2 + S * 4, T)
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
            emit(cfg, "ec_combine", timeit(lambda: B.ep_combine_expert_choice(recv, rt, lay, ew, out)),
                 S * H * 2 + T * H * 2 + S * 8 + (T + 1) * 4, T)
        if B.ep_get_device_error(lay) != 0:
            raise RuntimeError("device error flagged on workload %d" % wl)
    return 0


def main():
    args = parse()
    if args.workloads:
        return run_workload_table(args)
    if args.print_digests:
        print(json.dumps({k: source_digest(k) for k in KERNEL_SOURCES}))
        return 0
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
