"""Bench: MoE expert-parallel routing + layout -> dispatch -> combine on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--config prefill] [--impl ours|reference]

A step is one pass of the whole path over one batch: ep_get_layout (routing +
layout), ep_dispatch and ep_combine, with an identity expert in between.
The default workload is the prefill shape:
- 8 emulated ranks x 4096 tokens, H = 7168;
- 256 experts, group-limited top-8 (8 groups, keep 4);
- bf16 dispatch.
Its inputs (x 470 MB, receive rows 3.76 GB) exceed the 126 MB L2, so steps
run back to back with no flush. For workloads that fit in L2 (--config tiny
or decode) a 512 MB buffer is written between steps.

value = the step's algorithmic HBM bytes (layout + dispatch + combine) / step
time, in GB/s, summed over ranks. The timed region is K steps bracketed by a
barrier and a device sync, and the time is the max over ranks. Rank 0 prints
one JSON line.

N > 1 (under torchrun) runs the method one EP rank per GPU: R = N ranks, each
with the workload's T tokens per rank (weak scaling), the count all-gather
over NCCL, and dispatch / combine storing into and loading from the other
GPUs' receive arrays over NVLink (workspaces mapped through CUDA IPC). An NCCL all-to-all-v of
the same rows is timed beside it. --replicas runs N independent copies of the
emulated single-GPU job instead. --one-rank-per-gpu takes the per-GPU path on
one GPU too (R = 1).

--impl reference times the CPU oracle (the only reference this path has) on
all the host's cores, on rank 0, on a bounded sample of the same workload.
Other ranks exit 0.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from combine_top_group_b200 import metrics  # noqa: E402
from combine_top_group_b200 import workloads as wl  # noqa: E402

ORACLE_SAMPLE_T = 1024  # tokens per rank in the CPU oracle's bounded sample
# One metric string for both arms, so their lines compare directly.
METRIC = "routing+layout+dispatch+combine achieved HBM GB/s (algorithmic bytes / time)"
CPU_BASELINE_MIN_S = 10.0  # seconds of oracle work behind cpu_baseline


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="prefill", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0,
                    help="tokens per rank (0 = the workload's own); smaller cases for profiling")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--num-sms", type=int, default=0, help="SM cap for dispatch and combine (0 = all)")
    ap.add_argument("--fused-fp8-combine", action="store_true",
                    help="FP8 workloads: combine straight from the e4m3 rows (fused dequant)")
    ap.add_argument("--sweep-sms", action="store_true",
                    help="also time dispatch/combine under SM budgets 20, 1/4, 1/2, 3/4 and all SMs")
    ap.add_argument("--overlap", action="store_true",
                    help="also time dispatch+combine (20 SMs, own stream) against a concurrent bf16 GEMM")
    ap.add_argument("--dedup", action="store_true",
                    help="also time the deduplicated-receive pipeline (dispatch_dedup, permute, local_reduce, "
                         "combine_dedup) on the same workload")
    ap.add_argument("--graph", action="store_true",
                    help="also time the step captured in a CUDA graph (one replay per step)")
    ap.add_argument("--shard", action="store_true",
                    help="also time the one-rank-per-GPU calls, R ranks emulated on this GPU")
    ap.add_argument("--replicas", action="store_true",
                    help="--gpus N > 1: run N independent replicas of the emulated job instead of one EP rank per GPU")
    ap.add_argument("--one-rank-per-gpu", action="store_true",
                    help="run the one-EP-rank-per-GPU path even on one GPU (R = 1); the default for --gpus N > 1")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-copy-streams", type=int, default=1,
                    help="e2e: copy streams per direction (each copy split by rows)")
    return ap.parse_args(argv)


def workload_desc(w: wl.Workload) -> dict:
    return {"workload": w.describe(), "ranks_emulated": w.R, "tokens_per_rank": w.T, "hidden": w.H,
            "experts": w.E, "topk": w.K, "groups": w.G, "topk_groups": w.KG,
            "route": wl.ROUTE_NAMES[w.route], "dispatch": "fp8_e4m3" if w.fp8 else "bf16",
            "mask_frac": w.mask_frac}


# ---------------------------------------------------------------------------
# CPU oracle (test infrastructure) as the timed baseline
# ---------------------------------------------------------------------------

def oracle_sample(w: wl.Workload, seed: int = 0):
    """A bounded sample of the workload for the CPU oracle: the same shape with
    ORACLE_SAMPLE_T tokens per rank, and its seeded inputs."""
    ws = w.with_tokens(min(w.T, ORACLE_SAMPLE_T))
    return ws, wl.make_x(ws, seed), wl.make_logits(ws, seed)


def host_cores() -> int:
    """Cores this process may run on."""
    if hasattr(os, "sched_getaffinity"):
        return len(os.sched_getaffinity(0))
    return os.cpu_count() or 1


def oracle_step(ws: wl.Workload, x, logits, phases: dict | None = None, threads: int = 1):
    """One oracle pass (route, layout, dispatch, identity expert, combine) over
    the sample: single-threaded, or over token chunks on `threads` host
    threads (same C functions, identical outputs). Returns (seconds,
    algorithmic bytes); `phases` accumulates the seconds of each phase."""
    import oracle  # test infrastructure: only the CPU legs of the bench run it
    t0 = time.perf_counter()
    if threads > 1:
        res = oracle.run_path_parallel(x, logits, ws, threads, timings=phases)
    else:
        res = oracle.run_path(x, logits, ws, timings=phases)
    dt = time.perf_counter() - t0
    M = res["M"]
    return dt, metrics.layout_bytes(ws) + metrics.dispatch_bytes(ws, M) + metrics.combine_bytes(ws, M)


def host_cpu() -> dict:
    """The host's CPU model and logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu": model, "nproc": os.cpu_count()}


class OneCore:
    """Pins this process to one core of its allowed set while the oracle is
    timed (single-threaded C), then restores the previous set."""

    def __enter__(self):
        self.prev = None
        if hasattr(os, "sched_getaffinity"):
            try:
                self.prev = os.sched_getaffinity(0)
                os.sched_setaffinity(0, {min(self.prev)})
            except OSError:
                self.prev = None
        return self

    def __exit__(self, *exc):
        if self.prev is not None:
            os.sched_setaffinity(0, self.prev)
        return False


def _timed_oracle(ws, x, logits, threads: int, min_s: float):
    tot_t, tot_b, reps = 0.0, 0, 0
    phases: dict = {}
    while tot_t < min_s:
        dt, nb = oracle_step(ws, x, logits, phases, threads)
        tot_t += dt
        tot_b += nb
        reps += 1
    return tot_b / tot_t / 1e9, tot_t, reps, {k: v / reps * 1e3 for k, v in phases.items()}


def cpu_baseline(w: wl.Workload) -> dict:
    """The oracle on the host over the sample, repeated until CPU_BASELINE_MIN_S
    of work has been timed: on all the host's cores (token chunks on threads),
    and single-threaded pinned to one core."""
    ws, x, logits = oracle_sample(w)
    n = host_cores()
    v_all, t_all, r_all, ph_all = _timed_oracle(ws, x, logits, n, CPU_BASELINE_MIN_S)
    with OneCore():
        v_one, t_one, r_one, ph_one = _timed_oracle(ws, x, logits, 1, CPU_BASELINE_MIN_S)
    what = f"the whole path (route, layout, dispatch, identity expert, combine) over {ws.R}x{ws.T} tokens of " \
           f"the same shape"
    return {"value": v_all, "unit": "GB/s", "cores": n, "kind": "oracle",
            "sample": f"{r_all} passes of {what}; {t_all:.1f} s of C on {n} host threads (token chunks; "
                      f"mask and layout scan serial)",
            "phase_ms_per_pass": ph_all,
            "single_core": {"value": v_one, "unit": "GB/s", "cores": 1,
                            "sample": f"{r_one} passes, {t_one:.1f} s single-threaded, pinned to one core",
                            "phase_ms_per_pass": ph_one},
            "host": host_cpu()}


def run_reference(args, w: wl.Workload, rank: int, world: int):
    if rank != 0:
        return
    ws, x, logits = oracle_sample(w)
    tot_t, tot_b = 0.0, 0
    phases: dict = {}
    n = host_cores()
    for _ in range(args.warmup):
        oracle_step(ws, x, logits, threads=n)
    for _ in range(args.steps):
        dt, nb = oracle_step(ws, x, logits, phases, threads=n)
        tot_t += dt
        tot_b += nb
    value = tot_b / tot_t / 1e9
    line = {
        "impl": "reference", "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if not w.fp8 else "fp8_e4m3", "data": "synthetic",
        "config": {**workload_desc(w), "parallelism": f"{n} host threads", "combine_input": "bf16",
                   "sample_tokens_per_rank": ws.T,
                   "sample": f"each step runs the whole path over {ws.R}x{ws.T} of the workload's "
                             f"{w.R}x{w.T} tokens"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": n, "kind": "oracle",
                         "sample": f"each step: the whole path over {ws.R}x{ws.T} tokens of the same shape "
                                   f"(C over token chunks on {n} host threads; mask and layout scan serial)",
                         "phase_ms_per_pass": {k: v / args.steps * 1e3 for k, v in phases.items()},
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU path
# ---------------------------------------------------------------------------

def run_ours(args, w: wl.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from combine_top_group_b200 import ep, runner

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    pipe = runner.Pipeline(w, seed=rank, device=dev, num_sms=args.num_sms)
    fused = w.fp8 and args.fused_fp8_combine
    # identity expert for FP8 rows: y depends only on the (fixed) inputs, so it
    # is made once here, outside the timed region
    pipe.step(fused=True)
    if w.fp8 and not fused:
        pipe.identity_expert()
    if pipe.check_errors() != 0:
        raise RuntimeError("device error word set during set-up")
    M = pipe.moved_rows()
    bytes_layout = metrics.layout_bytes(w)
    bytes_dispatch = metrics.dispatch_bytes(w, M)
    bytes_combine = metrics.combine_bytes(w, M, fused_fp8=fused)
    bytes_step = bytes_layout + bytes_dispatch + bytes_combine

    fits_l2 = (w.N * w.H * 2 + M * w.H * (1 if w.fp8 else 2)) < 2 * 126 * 2 ** 20
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev) if fits_l2 else None

    def barrier():
        if world > 1:
            dist.barrier()

    props = torch.cuda.get_device_properties(dev)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    clk = metrics.ClockSampler(pci_bus_id=bus).start()
    for _ in range(args.warmup):
        if flush is not None:
            flush.fill_(1)
        pipe.step(fused=fused)
    torch.cuda.synchronize(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    t_host0 = time.perf_counter()
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        e = ev[i]
        e[0].record(stream)
        pipe.layout(stream)
        e[1].record(stream)
        pipe.dispatch(stream)
        e[2].record(stream)
        pipe.combine(fused=fused, stream=stream)
        e[3].record(stream)
        clk.sample_now()  # the host runs ahead of the device: this lands inside the timed region
    clk.sample_now(0.0)
    torch.cuda.synchronize(dev)
    clk.sample_now(0.0)
    t_host1 = time.perf_counter()
    barrier()
    clocks = clk.stop(t_host0, t_host1)
    if pipe.check_errors() != 0:
        raise RuntimeError("device error word set during the timed steps")

    t_layout = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_disp = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_comb = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_total = t_layout + t_disp + t_comb
    t_total, t_layout, t_disp, t_comb = metrics.max_over_ranks([t_total, t_layout, t_disp, t_comb], dev)
    K = args.steps
    value = world * bytes_step * K / t_total / 1e9

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(pipe, w, dev, stream, fused, bytes_step, steps=max(K, 8), world=world,
                          copy_streams=args.e2e_copy_streams)

    peak, peak_src = metrics.hbm_peak()
    d_avg, c_avg = t_disp / K, t_comb / K
    kern, k_bytes, k_time = (("dispatch", bytes_dispatch, d_avg) if d_avg >= c_avg
                             else ("combine", bytes_combine, c_avg))
    achieved = k_bytes / k_time / 1e9
    traffic = metrics.stored_traffic(kern, w.name)
    out = {
        "metric": METRIC,
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": t_total / K * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3" if w.fp8 else "bf16", "data": "synthetic",
        "config": {**workload_desc(w), "parallelism": f"replicas{world}" if world > 1 else "1gpu",
                   "num_sms": args.num_sms or "all", "combine_input": "fp8_fused" if fused else "bf16",
                   "l2": "512 MB flush between steps" if flush is not None else
                         "inputs larger than L2 (no flush)"},
        "layout_us": t_layout / K * 1e6, "dispatch_us": d_avg * 1e6, "combine_us": c_avg * 1e6,
        "dispatch_plus_combine_us": (d_avg + c_avg) * 1e6,
        "dispatch_gbs": bytes_dispatch / d_avg / 1e9, "combine_gbs": bytes_combine / c_avg / 1e9,
        "dispatch_frac_of_peak": bytes_dispatch / d_avg / 1e9 / peak,
        "combine_frac_of_peak": bytes_combine / c_avg / 1e9 / peak,
        "receive_rows": M,
        "algorithmic_bytes": {"layout": bytes_layout, "dispatch": bytes_dispatch, "combine": bytes_combine},
        "roofline": {"bound": "hbm", "kernel": kern, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": f"{peak_src} (hbm_gbs copy)"},
        "gpu_launches": 3 * K,  # layout, dispatch, combine: one kernel each
        "clocks": clocks,
    }
    why = metrics.clocks_rejected(clocks)
    if why:
        out["clocks_rejected"] = why
    if e2e is not None:
        out["e2e"] = e2e
    if args.sweep_sms:
        out["sms_sweep"] = sweep_sms(pipe, w, fused, stream, bytes_dispatch, bytes_combine, props.multi_processor_count)
    if args.overlap:
        out["overlap"] = measure_overlap(pipe, w, dev, fused)
    if args.dedup:
        out["dedup"] = measure_dedup(w, rank, dev, fused, steps=min(args.steps, 10))
    if args.graph:
        t = time_graph(lambda: pipe.step(fused=fused), dev, flush, steps=args.steps)
        out["graph"] = {"step_us": t * 1e6, "value": bytes_step / t / 1e9, "unit": "GB/s",
                        "launches_per_step": 3, "steps": args.steps}
    if args.shard:
        out["shard"] = (measure_shard(pipe, w, dev, fused, bytes_dispatch, bytes_combine, flush,
                                      steps=min(args.steps, 10), graph=args.graph)
                        if world == 1 else {"skipped": "the emulated ranks run on one GPU (--gpus 1)"})
    ep.ep_buffer_set_num_sms(pipe.buf, args.num_sms)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(out), flush=True)


def sweep_sms(pipe, w, fused, stream, bytes_dispatch, bytes_combine, sm_count, steps=10):
    """Dispatch and combine alone under SM budgets (Buffer.set_num_sms):
    DeepEP's default 20, then 1/4, 1/2, 3/4 and all of the SMs."""
    import torch

    from combine_top_group_b200 import ep
    rows = []
    for n in (20, sm_count // 4, sm_count // 2, 3 * sm_count // 4, sm_count):
        ep.ep_buffer_set_num_sms(pipe.buf, n)
        pipe.dispatch(stream)
        pipe.combine(fused=fused, stream=stream)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        for _ in range(steps):
            pipe.dispatch(stream)
        ev[1].record(stream)
        for _ in range(steps):
            pipe.combine(fused=fused, stream=stream)
        ev[2].record(stream)
        torch.cuda.synchronize()
        d = ev[0].elapsed_time(ev[1]) / steps / 1e3
        c = ev[1].elapsed_time(ev[2]) / steps / 1e3
        rows.append({"num_sms": n, "dispatch_us": d * 1e6, "dispatch_gbs": bytes_dispatch / d / 1e9,
                     "combine_us": c * 1e6, "combine_gbs": bytes_combine / c / 1e9})
    return rows


def measure_overlap(pipe, w, dev, fused, comm_sms=20, reps=5):
    """Compute/communication overlap (DeepEP overlap notes, §节点内通信):
    dispatch + combine capped at `comm_sms` SMs on a communication stream, next
    to a bf16 GEMM on a compute stream. The GEMM is a cuBLAS stand-in for the
    expert work and is not part of the path. Reports both times alone and
    together, and how much of the shorter one the overlap hid."""
    import torch

    from combine_top_group_b200 import ep
    comp = torch.cuda.Stream(dev)
    comm = torch.cuda.Stream(dev)
    a = torch.randn(8192, 7168, dtype=torch.bfloat16, device=dev)
    b = torch.randn(7168, 8192, dtype=torch.bfloat16, device=dev)
    ep.ep_buffer_set_num_sms(pipe.buf, comm_sms)

    def gemm():
        with torch.cuda.stream(comp):
            for _ in range(reps):
                torch.matmul(a, b)

    def comms():
        for _ in range(reps):
            pipe.dispatch(comm)
            pipe.combine(fused=fused, stream=comm)

    def timed(fn_list):
        start = torch.cuda.Event(enable_timing=True)
        start.record(torch.cuda.current_stream(dev))
        ends = []
        for st, fn in fn_list:
            st.wait_event(start)
            fn()
            e = torch.cuda.Event(enable_timing=True)
            e.record(st)
            ends.append(e)
        torch.cuda.synchronize(dev)
        return max(start.elapsed_time(e) for e in ends) / reps

    timed([(comp, gemm), (comm, comms)])  # warm-up
    t_gemm = timed([(comp, gemm)])
    t_comm = timed([(comm, comms)])
    t_both = timed([(comp, gemm), (comm, comms)])
    ep.ep_buffer_set_num_sms(pipe.buf, 0)
    t_comm_all = timed([(comm, comms)])
    hidden = (t_gemm + t_comm - t_both) / min(t_gemm, t_comm)
    return {"comm_sms": comm_sms, "gemm_ms": t_gemm, "comm_ms": t_comm, "comm_ms_all_sms": t_comm_all,
            "together_ms": t_both, "serial_ms": t_gemm + t_comm, "hidden_frac_of_shorter": hidden,
            "gemm": "bf16 8192x7168 @ 7168x8192 (cuBLAS stand-in for expert compute)"}


def measure_dedup(w, seed, dev, fused, steps):
    """Deduplicated receive (one row per token and destination rank), timed
    kernel by kernel. rows_dedup / rows_expert is the share of expert rows
    that would cross the links in a real multi-GPU all-to-all."""
    import torch

    from combine_top_group_b200 import runner
    pipe = runner.Pipeline(w, seed=seed, device=dev, dedup=True)
    stream = torch.cuda.current_stream(dev)
    pipe.layout(stream)
    pipe.dispatch_dedup(stream)
    pipe.permute(stream)
    if w.fp8 and not fused:
        pipe.identity_expert()
    pipe.local_reduce(fused=fused, stream=stream)
    pipe.combine_dedup(stream)
    if pipe.check_errors() != 0:
        raise RuntimeError("device error word set in the dedup pipeline")
    D, M = pipe.dedup_rows(), pipe.moved_rows()
    names = ["layout", "dispatch_dedup", "permute", "local_reduce", "combine_dedup"]
    calls = [lambda: pipe.layout(stream), lambda: pipe.dispatch_dedup(stream), lambda: pipe.permute(stream),
             lambda: pipe.local_reduce(fused=fused, stream=stream), lambda: pipe.combine_dedup(stream)]
    tot = [0.0] * len(calls)
    for _ in range(steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        ev[0].record(stream)
        for i, c in enumerate(calls):
            c()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        for i in range(len(calls)):
            tot[i] += ev[i].elapsed_time(ev[i + 1]) / 1e3
    b = 1 if w.fp8 else 2
    yb = (M * w.H + M * (w.H // 128) * 4) if (w.fp8 and fused) else M * w.H * 2
    scales = (w.H // 128) * 4 if w.fp8 else 0
    nbytes = [metrics.layout_bytes(w),
              w.N * w.H * 2 + w.N * w.K * 8 + D * (w.H * b + scales + 4 + w.K * 8),  # x, topk, rows + ids + local top-k
              D * (w.H * b + scales + w.K * 8 + 4) + M * (w.H * b + scales + 8),     # dedup rows in, expert rows out
              yb + D * w.K * 8 + D * w.H * 2,                                        # expert outputs in, partials out
              D * w.H * 2 + w.N * w.H * 2]                                           # partials in, out
    res = {"rows_dedup": D, "rows_expert": M, "dedup_ratio": D / M if M else None, "steps": steps}
    for n, t, nb in zip(names, tot, nbytes):
        res[n + "_us"] = t / steps * 1e6
        res[n + "_gbs"] = nb / (t / steps) / 1e9
    del pipe
    return res


def time_graph(step, dev, flush, steps):
    """Seconds per step of `step` captured once in a CUDA graph and replayed:
    every launch of the step is enqueued by one graph launch, so host
    overhead between kernels drops out. Events bracket each replay; the L2
    flush (if any) runs between replays, outside them."""
    import torch
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()  # warm-up on the capture stream's side
    torch.cuda.current_stream(dev).wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        if flush is not None:
            flush.fill_(1)
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize(dev)
    t = sum(a.elapsed_time(b) for a, b in ev) / 1e3 / steps
    del g
    return t


def measure_shard(pipe, w, dev, fused, bytes_dispatch, bytes_combine, flush, steps, graph=False):
    """The one-rank-per-GPU calls (EP_FLAG_SHARD) with all R ranks emulated on
    this GPU: per step R layouts, the count all-gather (device copies), R
    placements, R dispatches and R combines, each phase timed with events.
    The same rows move as in the single-buffer path, so the same algorithmic
    bytes apply. Eagerly, the R small launches per phase are host-bound;
    with graph=True the whole step is also timed as one CUDA graph replay."""
    import torch

    from combine_top_group_b200 import shard
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(pipe.out)
    em = shard.EmulatedRanks(w, pipe.x, pipe.logits, out)
    em.step(stream)
    if w.fp8 and not fused:
        em.identity_expert()
    if em.check_errors() != 0:
        raise RuntimeError("device error word set in the one-rank-per-GPU path")
    same = bool(torch.equal(out.view(torch.int16), pipe.out.view(torch.int16))) if not w.fp8 or fused else None
    names = ["layout", "exchange", "place", "dispatch", "combine"]
    calls = [lambda: em.layout(stream), lambda: em.exchange(stream), lambda: em.place(stream),
             lambda: em.dispatch(stream), lambda: em.combine(stream)]
    tot = [0.0] * len(calls)
    for _ in range(steps):
        if flush is not None:
            flush.fill_(1)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        ev[0].record(stream)
        for i, c in enumerate(calls):
            c()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        for i in range(len(calls)):
            tot[i] += ev[i].elapsed_time(ev[i + 1]) / 1e3
    res = {"ranks": w.R, "steps": steps, "launches_per_step": 4 * w.R + 1 + w.R,
           "out_equals_single_buffer": same, "received_rows": em.received_rows()}
    for n, t in zip(names, tot):
        res[n + "_us"] = t / steps * 1e6
    res["dispatch_gbs"] = bytes_dispatch / (tot[3] / steps) / 1e9
    res["combine_gbs"] = bytes_combine / (tot[4] / steps) / 1e9
    res["step_us"] = sum(tot) / steps * 1e6
    if graph:
        res["graph_step_us"] = time_graph(lambda: em.step(None), dev, flush, steps) * 1e6
    del em
    return res


def measure_e2e(pipe, w, dev, stream, fused, bytes_step, steps, world, copy_streams=1):
    """Same metric, through the C ABI, with the step's inputs copied in from
    pinned host memory and its result copied back, inside the timed region.

    Steps are double-buffered: device x / logits / out have two slots. The
    host-to-device copies run on their own copy streams and the device-to-host
    copies on others, so step i+1's inputs and step i-1's result cross PCIe
    (full duplex) while step i computes. With copy_streams > 1 each copy is
    split by rows over that many streams per direction. Every step still
    copies all of its inputs in and its whole result out."""
    import torch
    import torch.distributed as dist
    x_h = pipe.x.cpu().pin_memory()
    l_h = pipe.logits.cpu().pin_memory()
    out_h = torch.empty(pipe.out.shape, dtype=pipe.out.dtype).pin_memory()
    h2d = x_h.numel() * x_h.element_size() + l_h.numel() * l_h.element_size()
    d2h = out_h.numel() * out_h.element_size()
    xs = [pipe.x, torch.empty_like(pipe.x)]
    ls = [pipe.logits, torch.empty_like(pipe.logits)]
    outs = [pipe.out, torch.empty_like(pipe.out)]
    keep = (pipe.x, pipe.logits, pipe.out)
    C = max(1, copy_streams)
    s_in = [torch.cuda.Stream(dev) for _ in range(C)]
    s_out = [torch.cuda.Stream(dev) for _ in range(C)]

    def rows(t, c):  # row range c of C
        n = t.shape[0]
        return t[n * c // C:n * (c + 1) // C]

    def ev():
        return torch.cuda.Event()

    in_done = [[ev() for _ in range(C)] for _ in range(2)]
    out_done = [[ev() for _ in range(C)] for _ in range(2)]
    comp_done = [ev(), ev()]

    def one(i):
        k = i % 2
        for c in range(C):
            s_in[c].wait_event(comp_done[k])  # step i-2 has finished reading slot k's inputs
            with torch.cuda.stream(s_in[c]):
                rows(xs[k], c).copy_(rows(x_h, c), non_blocking=True)
                rows(ls[k], c).copy_(rows(l_h, c), non_blocking=True)
            in_done[k][c].record(s_in[c])
            stream.wait_event(in_done[k][c])
            stream.wait_event(out_done[k][c])  # step i-2's result has left slot k
        pipe.x, pipe.logits, pipe.out = xs[k], ls[k], outs[k]
        pipe.layout(stream)
        pipe.dispatch(stream)
        if w.fp8 and not fused:
            pipe.combine(fused=False, stream=stream)  # y made once from the same inputs
        else:
            pipe.combine(fused=fused, stream=stream)
        comp_done[k].record(stream)
        for c in range(C):
            s_out[c].wait_event(comp_done[k])
            with torch.cuda.stream(s_out[c]):
                rows(out_h, c).copy_(rows(outs[k], c), non_blocking=True)
            out_done[k][c].record(s_out[c])

    try:
        for i in range(2):  # warm-up; records every event once
            one(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for c in range(C):
            s_in[c].wait_event(s)
        for i in range(steps):
            one(i)
        for k in range(2):
            for c in range(C):
                stream.wait_event(out_done[k][c])
        e.record(stream)
        torch.cuda.synchronize(dev)
    finally:
        pipe.x, pipe.logits, pipe.out = keep
    t = metrics.max_over_ranks([s.elapsed_time(e) / 1e3], dev)[0]
    return {"value": world * bytes_step * steps / t / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": t / steps * 1e3,
            "copies": f"pinned host buffers; H2D and D2H each on {C} copy stream(s), double-buffered across steps"}


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def ep_workload(w: wl.Workload, world: int) -> wl.Workload:
    """The workload as a node runs it: R = world ranks (one per GPU), the
    same T tokens per rank, experts, routing and hidden size."""
    import dataclasses
    if w.low_latency:
        raise SystemExit("the one-rank-per-GPU path uses the standard receive layout")
    if w.E % world:
        raise SystemExit(f"E={w.E} is not a multiple of {world} ranks")
    return dataclasses.replace(w, R=world)


def run_ep(args, w0: wl.Workload, rank: int, world: int, local_rank: int):
    """One EP rank per GPU (shard.DistributedRank): this process routes its own
    T tokens, all-gathers the count rows, and dispatch / combine store into and
    load from every rank's receive arrays (peer memory over NVLink). Phases are
    timed with events on the launching stream; the barriers between them are
    stream-ordered NCCL all-reduces, included in the phase that waits on them.
    FP8 workloads combine straight from the e4m3 rows (fused dequantisation)."""
    import torch
    import torch.distributed as dist

    from combine_top_group_b200 import shard

    w = ep_workload(w0, world)
    T, H = w.T, w.H
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    drv = shard.DistributedRank(w, dev, num_sms=args.num_sms)
    xs = wl.make_x(w, 0, rows=slice(rank * T, (rank + 1) * T))
    x = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).to(dev)
    logits = torch.from_numpy(np.ascontiguousarray(wl.make_logits(w, 0)[rank * T:(rank + 1) * T])).to(dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        drv.layout(logits)
        drv.exchange()
        drv.place()
        if ev is not None:
            ev[1].record(stream)
        drv.barrier()  # every rank has finished reading the previous step's rows
        drv.dispatch(x)
        if ev is not None:
            ev[2].record(stream)
        drv.barrier()  # every rank's rows are written (identity experts)
        drv.combine(out)
        if ev is not None:
            ev[3].record(stream)

    step()
    torch.cuda.synchronize(dev)
    if drv.check_errors() != 0:
        raise RuntimeError("device error word set during set-up")
    check = ep_output_check(w, x, out, drv)
    send, recv = drv.alltoallv_splits()
    M_s = sum(send)  # rows this rank's tokens send
    remote = M_s - send[rank]  # of which to other GPUs
    b = 1 if w.fp8 else 2
    row_b = H * b + ((H // 128) * 4 if w.fp8 else 0)
    bytes_layout = metrics.layout_bytes(w, N=T)
    bytes_dispatch = metrics.dispatch_bytes(w, M_s, N=T)
    bytes_combine = metrics.combine_bytes(w, M_s, fused_fp8=w.fp8, N=T)
    totals = metrics.sum_over_ranks([bytes_layout, bytes_dispatch, bytes_combine, remote * (row_b + 8),
                                     remote * row_b], dev)
    bytes_step = sum(totals[:3])

    props = torch.cuda.get_device_properties(dev)
    bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    clk = metrics.ClockSampler(pci_bus_id=bus).start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_host0 = time.perf_counter()
    for i in range(K):
        step(ev[i])
        clk.sample_now()
    clk.sample_now(0.0)
    torch.cuda.synchronize(dev)
    clk.sample_now(0.0)
    t_host1 = time.perf_counter()
    dist.barrier()
    clocks = clk.stop(t_host0, t_host1)
    if drv.check_errors() != 0:
        raise RuntimeError("device error word set during the timed steps")
    t_lay = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_disp = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_comb = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_total, t_lay, t_disp, t_comb = metrics.max_over_ranks([t_lay + t_disp + t_comb, t_lay, t_disp, t_comb], dev)
    value = bytes_step * K / t_total / 1e9

    nccl = nccl_alltoallv_baseline(drv, w, send, recv, dev, reps=max(3, min(K, 10)))
    e2e = None if args.no_e2e else measure_e2e_ep(step, x, logits, out, dev, stream, bytes_step,
                                                  steps=max(K, 5))
    d_avg, c_avg = t_disp / K, t_comb / K
    peak_hbm, peak_src = metrics.hbm_peak()
    if world > 1:
        # bound: the rows that cross NVLink, per direction per GPU, at the
        # measured peer-copy bandwidth
        nv_bytes = totals[3] / world
        roof = {"bound": "nvlink", "kernel": "dispatch", "achieved": nv_bytes / d_avg / 1e9,
                "peak": metrics.NVLINK_PEER_GBS, "unit": "GB/s",
                "frac": nv_bytes / d_avg / 1e9 / metrics.NVLINK_PEER_GBS, "traffic": None,
                "peak_source": "measured peer copy per direction (NVLink 5)"}
    else:
        roof = {"bound": "hbm", "kernel": "dispatch", "achieved": totals[1] / d_avg / 1e9, "peak": peak_hbm,
                "unit": "GB/s", "frac": totals[1] / d_avg / 1e9 / peak_hbm, "traffic": None,
                "peak_source": f"{peak_src} (hbm_gbs copy)"}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": t_total / K * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3" if w.fp8 else "bf16", "data": "synthetic",
        "config": {**{k: v for k, v in workload_desc(w).items() if k != "ranks_emulated"}, "ep_ranks": world,
                   "parallelism": f"ep{world}: one EP rank per GPU, peer stores/loads "
                                                      f"through IPC-mapped workspaces, NCCL count all-gather",
                   "num_sms": args.num_sms or "all", "combine_input": "fp8_fused" if w.fp8 else "bf16",
                   "l2": "inputs larger than L2 (no flush)" if T * H * 2 * w.K > 2 * 126 * 2 ** 20 else
                         "no flush (small per-rank batch)"},
        "layout_us": t_lay / K * 1e6, "dispatch_us": d_avg * 1e6, "combine_us": c_avg * 1e6,
        "dispatch_plus_combine_us": (d_avg + c_avg) * 1e6,
        "phases": "layout = route + count all-gather + place; dispatch and combine each include the "
                  "cross-rank barrier before them",
        "dispatch_gbs": totals[1] / world / d_avg / 1e9, "combine_gbs": totals[2] / world / c_avg / 1e9,
        "rows_sent_per_rank": M_s, "rows_to_other_gpus_per_rank": remote,
        "nvlink_bytes_per_step": {"dispatch": totals[3], "combine": totals[4]},
        "algorithmic_bytes": {"layout": totals[0], "dispatch": totals[1], "combine": totals[2]},
        "roofline": roof, "nccl_alltoallv": nccl, "output_check": check,
        "gpu_launches": 4 * K,  # layout, place, dispatch, combine per step (NCCL's own kernels not counted)
        "clocks": clocks,
    }
    why = metrics.clocks_rejected(clocks)
    if why:
        line["clocks_rejected"] = why
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0:
        print(json.dumps(line), flush=True)


def ep_output_check(w, x, out, drv) -> dict:
    """A property that holds at any size, checked on the device after a step
    with identity experts: each token's output is its input scaled by the sum
    of its top-k weights, out[t] = x[t] * sum_k w[t,k], within the bf16
    combine tolerance (2^-7 |ref| + 1e-3), or the FP8 round trip's (2^-4
    relative, e4m3 having 3 mantissa bits). Rows lost or misplaced on the
    way to another GPU and back break it."""
    import torch
    lay = drv.ep.ep_buffer_layout(drv.buf, w.T)
    ref = x.float() * lay["topk_w"].sum(dim=1, keepdim=True)
    err = (out.float() - ref).abs()
    rel = 2.0 ** -4 + 2.0 ** -7 if w.fp8 else 2.0 ** -7
    bad = int((err > rel * ref.abs() + 1e-3).sum().item())
    ok = bad == 0
    if not ok:
        raise RuntimeError(f"output check failed on {bad} elements (max err {float(err.max()):.3g})")
    return {"passed": True, "elements": int(out.numel()), "rule": "out = x * sum_k w within tolerance"}


def nccl_alltoallv_baseline(drv, w, send, recv, dev, reps: int) -> dict:
    """NCCL all-to-all-v moving the same rows between the ranks: this rank's
    rows grouped by destination (split sizes from the exchanged counts), then
    the reverse exchange for the combine. Only the collectives are timed: no
    packing, no quantisation, no weighted sum."""
    import torch
    import torch.distributed as dist
    dt = torch.uint8 if w.fp8 else torch.bfloat16
    cols = w.H + (w.H // 128) * 4 if w.fp8 else w.H  # FP8 rows carry their scales
    sbuf = torch.empty(max(sum(send), 1), cols, dtype=dt, device=dev)
    rbuf = torch.empty(max(sum(recv), 1), cols, dtype=dt, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        dist.all_to_all_single(rbuf[:sum(recv)], sbuf[:sum(send)], recv, send)

    def bwd():
        dist.all_to_all_single(sbuf[:sum(send)], rbuf[:sum(recv)], send, recv)

    fwd()
    bwd()
    torch.cuda.synchronize(dev)
    dist.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(stream)
    for _ in range(reps):
        fwd()
    ev[1].record(stream)
    for _ in range(reps):
        bwd()
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    t_f, t_b = metrics.max_over_ranks([ev[0].elapsed_time(ev[1]) / 1e3 / reps,
                                       ev[1].elapsed_time(ev[2]) / 1e3 / reps], dev)
    row_bytes = cols * (1 if w.fp8 else 2)
    total = metrics.sum_over_ranks([sum(send) * row_bytes], dev)[0]
    return {"dispatch_direction_us": t_f * 1e6, "combine_direction_us": t_b * 1e6,
            "bytes_moved": total, "reps": reps,
            "what": "torch.distributed.all_to_all_single (NCCL) of the same rows, split sizes from the "
                    "exchanged counts; collectives only"}


def measure_e2e_ep(step, x, logits, out, dev, stream, bytes_step, steps: int) -> dict:
    """The EP step end to end through the public calls: every step copies
    this rank's x and logits in from pinned host memory and its output back,
    on the launching stream, inside the timed region."""
    import torch
    x_h = x.cpu().pin_memory()
    l_h = logits.cpu().pin_memory()
    o_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def one():
        x.copy_(x_h, non_blocking=True)
        logits.copy_(l_h, non_blocking=True)
        step()
        o_h.copy_(out, non_blocking=True)

    one()
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        one()
    e.record(stream)
    torch.cuda.synchronize(dev)
    t = metrics.max_over_ranks([s.elapsed_time(e) / 1e3], dev)[0]
    return {"value": bytes_step * steps / t / 1e9, "unit": "GB/s",
            "h2d_bytes_per_step": x_h.numel() * 2 + l_h.numel() * 4, "d2h_bytes_per_step": o_h.numel() * 2,
            "steps": steps, "ms_per_step": t / steps * 1e3,
            "copies": "pinned host buffers, copies on the launching stream (per rank)"}


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.WORKLOADS[args.config]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    import datetime

    import torch
    import torch.distributed as dist
    per_gpu = args.one_rank_per_gpu or (world > 1 and not args.replicas)
    if world > 1 or per_gpu:
        torch.cuda.set_device(local_rank)
        kw = {}
        if world == 1 and "MASTER_ADDR" not in os.environ:
            kw = dict(init_method=f"tcp://127.0.0.1:{free_port()}", rank=0, world_size=1)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank), **kw)
    try:
        if per_gpu:
            run_ep(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
