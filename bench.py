"""Benchmark: Gaussian kernel-sum throughput (G pairs/s) on B200, with the
roofline fraction of the dominant kernel and the CPU oracle as the baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole hot path of the workload over its seeded
synthetic inputs (already resident in HBM).  Default workload: ``d3_1m_lse``
(B=1, M=N=1,000,000, D=3, C=1, fp32, tau=100, x,y ~ U[0,1)^3, w ~ U(0.5,1.5)):
one step is the Gaussian kernel sum and its log-sum-exp over the same inputs,
the largest single-GPU workload (the 1M-point Gaussian product of "Kernel
matrix reduction", Variants, plus the log-sum-exp reduction of its Overview).
Under torchrun (N > 1) every rank runs its own independent problem of that
size (rank-specific query points, same sources): rows are independent, so
there is no data-path collective, and throughput scales weakly; the time is
the maximum over ranks.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on
the launching stream, with a 256 MiB write between steps to flush the 126 MB L2
(the inputs are smaller than L2); barrier + synchronize around the timed loop.
SM clocks and throttle reasons are sampled with nvidia-smi during the loop.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

# MUFU ex2 throughput: 16 results / clock / SM (4 per SM sub-partition); every
# pair of the small-D and tensor-core paths costs exactly one ex2 on the MUFU
# pipe, so the ALU roofline in pairs/s is 16 * SMs * clock.
EX2_PER_CLK_PER_SM = 16
PUBLISHED = {  # context only: the pages' number for the same workload, another GPU
    "d3_100k": {"value": 1e10 / 15.0e-3 / 1e9,
                "source": "KeOps Gaussian product, 100k points, 15.0 ms on an RTX 2080 Ti"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="d3_1m_lse", choices=sorted(synth.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e-single-steps", type=int, default=5,
                    help="steps of the one-call-at-a-time end-to-end figure (one stream, no overlap)")
    ap.add_argument("--no-launch-count", action="store_true",
                    help="skip the profiler-based kernel count (use under ncu)")
    ap.add_argument("--clock-log", default=None,
                    help="CSV of the nvidia-smi clock samples (default: a file under the temp directory)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch each timed step from the host instead of replaying it from a "
                         "CUDA graph captured after the warm-up")
    ap.add_argument("--two-call", action="store_true",
                    help="forward + backward workloads: time gauss_sum_fwd_saved then "
                         "gauss_sum_bwd_saved (two sweeps, g not needed by the forward) instead "
                         "of the one-call gauss_sum_fwd_bwd")
    ap.add_argument("--sharded", action="store_true",
                    help="one problem of the workload's size split over the ranks by rows and "
                         "sources (strong scaling; the sources are all-gathered every step)")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_init(n_gpus, need_group=False):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1 or need_group:
        if world == 1:   # a one-rank group, for the collectives of the sharded mode
            import socket
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                with socket.socket() as sk:
                    sk.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(value, pg, device):
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, path):
        self.index, self.path, self.proc = index, path, None

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if getattr(self, "f", None):
            self.f.close()

    def summary(self):
        try:
            rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        except OSError:
            rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], None, set()
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ workloads
def sharded_step_fn(w, d, counts):
    """One pass of the hot path for this rank's shard of one problem (counts: the
    ranks' row and source counts, exchanged once before timing)."""
    from pairwise_reductions_b200 import sharded
    tau = d["tau"]
    rc, sc = counts

    def run():
        if "sum" in w.ops:
            d["out_sum"] = sharded.sharded_sum_fwd(d["x"], d["y"], d["w"], tau, src_counts=sc)
        if "lse" in w.ops:
            d["out_lse"] = sharded.sharded_lse_fwd(d["x"], d["y"], d["w"], tau, src_counts=sc)
        if "bwd" in w.ops:
            sharded.sharded_sum_bwd(d["x"], d["y"], d["w"], d["g"], tau, row_counts=rc,
                                    src_counts=sc)
    return run


def shard_of(inp, rank, world):
    """Contiguous row and source slices of the whole problem for this rank."""
    def sl(n):
        lo = n * rank // world
        return slice(lo, n * (rank + 1) // world)
    rows, srcs = sl(inp["x"].shape[1]), sl(inp["y"].shape[1])
    out = dict(inp)
    out["x"] = inp["x"][:, rows].contiguous()
    out["y"] = inp["y"][:, srcs].contiguous()
    out["w"] = inp["w"][:, srcs].contiguous()
    if "g" in inp:
        out["g"] = inp["g"][:, rows].contiguous()
    return out


def step_fn(gs, w, d, ws, outs, two_call=False):
    """Return a closure running one pass of the workload's hot path."""
    tau = d["tau"]
    ops = w.ops

    def run(mid=None):
        if "sum" in ops and "bwd" in ops and not two_call:
            # forward and backward in one call (g given up front)
            gs.gauss_sum_fwd_bwd(d["x"], d["y"], d["w"], d["g"], tau, out=outs["sum"],
                                 grad_x=outs["gx"], grad_w=outs["gw"], workspace=ws)
        elif "sum" in ops and "bwd" in ops:
            # forward that keeps the x-gradient sums, then the backward from them
            # (mid: an event recorded between the two, for the per-part times)
            gs.gauss_sum_fwd_saved(d["x"], d["y"], d["w"], tau, out=outs["sum"],
                                   saved=outs["saved"], workspace=ws)
            if mid is not None:
                mid.record()
            gs.gauss_sum_bwd_saved(d["x"], d["y"], d["w"], d["g"], outs["saved"], tau, workspace=ws)
        elif "sum" in ops:
            gs.gauss_sum_fwd(d["x"], d["y"], d["w"], tau, out=outs["sum"], workspace=ws)
        elif "bwd" in ops:
            gs.gauss_sum_bwd(d["x"], d["y"], d["w"], d["g"], tau, workspace=ws)
        if "lse" in ops:
            gs.gauss_lse_fwd(d["x"], d["y"], d["w"], tau, out=outs["lse"], workspace=ws)
    return run


def pairs_per_step(w):
    """Pairs (B*M*N) one step reduces, per output: the sum and the log-sum-exp count
    once each; a forward + backward step counts its pairs once (the combined figure
    B*M*N / (t_fwd + t_bwd)); a backward alone counts once."""
    per = w.pairs
    return per * (("sum" in w.ops or "bwd" in w.ops) + ("lse" in w.ops))


def fused_fwd_bwd(w):
    """Whether gauss_sum_fwd_bwd evaluates each kernel value once for this
    workload (fp16 / bf16, C = 1, D <= 47); else it runs two sweeps."""
    return w.dtype != "f32" and w.C == 1 and w.D <= 47


def kernel_evals_per_step(w, two_call=False):
    """Kernel evaluations (exponentials) one step performs: one sweep per sum or
    log-sum-exp; the forward + backward step runs one sweep in one call where it
    fuses, else two (the forward that keeps the x-gradient sums, and the
    grad_w pass)."""
    if "sum" in w.ops and "bwd" in w.ops:
        return w.pairs * (1 if (fused_fwd_bwd(w) and not two_call) else 2) + \
            w.pairs * ("lse" in w.ops)
    return w.pairs * (("sum" in w.ops) + ("lse" in w.ops) + ("bwd" in w.ops))


def tensor_flops_per_step(w):
    """Tensor-core FLOPs (2 per multiply-add) one step needs by the method's own
    arithmetic, or 0 where the pair work runs on the CUDA cores (fp32, D <= 8) or
    the step mixes passes (the backward workloads report the MUFU bound).
    fp32 inputs, D > 8: each value product is three fp16-part products, so the
    similarity costs 3 * 2D a pair, and P.v with values on the tensor cores (more
    than three channels) 3 * 2C a pair.  fp16 / bf16: the similarity on rows
    augmented by the two norm terms, 2 (D + 2) a pair, and P.v 2C a pair for more
    than one channel (one channel is summed in registers); their log-sum-exp
    takes the unsplit rows, 2D a pair."""
    if "bwd" in w.ops or (w.dtype == "f32" and w.D <= 8):
        return 0
    if w.dtype == "f32":
        sum_pp = 6 * w.D + (6 * w.C if w.C > 3 else 0)
        lse_pp = 6 * w.D
    else:
        sum_pp = 2 * (w.D + 2) + (2 * w.C if w.C > 1 else 0)
        lse_pp = 2 * w.D
    return w.pairs * (sum_pp * ("sum" in w.ops) + lse_pp * ("lse" in w.ops))


def launches_per_step(gs, run):
    """Kernels one step launches, counted by the CUDA profiler (names prove they are ours)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA
             and ("gs::" in e.name or "gauss" in e.name or "kernel" in e.name)]
    return len(names), sorted(set(names))


# ------------------------------------------------------------------ ncu traffic of the dominant kernel
def dominant(w):
    """(kernel, source file) that does the pair work of a workload."""
    if w.dtype != "f32":
        return "tc_gauss_kernel", "tc_sm100.cu"
    return ("sd_kernel", "small_d.cu") if w.D <= 8 else ("tc_f32_kernel", "tc_f32_sm100.cu")


def traffic_per_launch(w):
    """DRAM bytes (read + write) per launch of the dominant kernel from the committed ncu
    summary, or None when there is none for this workload or the kernel source changed since."""
    import hashlib
    kernel, src = dominant(w)
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None, kernel
    cur = hashlib.sha256(open(os.path.join(ROOT, "pairwise_reductions_b200", "csrc", src), "rb").read())
    for line in lines:
        f = line.split()
        if len(f) == 6 and not line.startswith("#") and f[0] == kernel and f[1] == w.name:
            if f[4] == src and cur.hexdigest().startswith(f[5]):
                return int(f[2]) + int(f[3]), kernel
    return None, kernel


# ------------------------------------------------------------------ CPU oracle baseline
def oracle_sample(w, inp, seconds, seed=1234):
    """Time the oracle as it stands on a bounded row sample of the workload."""
    import oracle
    import numpy as np
    x, y, wt = (synth.as_f64(inp[k]) for k in ("x", "y", "w"))
    g = synth.as_f64(inp["g"]) if "g" in inp else None

    def run(rows):
        t0 = time.perf_counter()
        if "sum" in w.ops:
            oracle.gauss_sum(x, y, wt, w.tau, rows=rows)
        if "lse" in w.ops:
            oracle.gauss_lse(x, y, wt, w.tau, rows=rows)
        if "bwd" in w.ops:
            oracle.gauss_sum_bwd(x, y, wt, g, w.tau, rows=rows, wrows=rows % w.N)
        return time.perf_counter() - t0

    # size the sample in two probes: 16 rows carry the start-up costs, so a
    # second probe of about a tenth of the target corrects the per-row time
    probe = synth.sample_rows(w.M, 16, seed).numpy()
    t = max(run(probe), 1e-3)
    n1 = int(min(w.M, max(16, 16 * 0.1 * seconds / t)))
    if n1 > 16:
        t1 = max(run(synth.sample_rows(w.M, n1, seed).numpy()), 1e-3)
        n = int(min(w.M, max(16, n1 * seconds / t1)))
    else:
        n = int(min(w.M, max(16, 16 * seconds / t)))
    rows = synth.sample_rows(w.M, n, seed).numpy()
    dt = run(rows)
    pairs = w.B * n * w.N * (("sum" in w.ops or "bwd" in w.ops) + ("lse" in w.ops))
    return {"value": pairs / dt / 1e9, "unit": "G pairs/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"{n} of {w.M} query rows x all {w.N} sources, B={w.B}, same seeded inputs"}, rows


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.make_inputs(w)
    # the whole timed loop takes about --cpu-seconds: each step a row sample of at
    # least 0.1 s of oracle work (~2e8 pairs on 16 cores), so even thousands of
    # steps end within minutes
    per_step = args.cpu_seconds / max(args.steps, 1)
    import oracle
    base, rows = oracle_sample(w, inp, max(per_step, 0.1))
    x, y, wt = (synth.as_f64(inp[k]) for k in ("x", "y", "w"))
    g = synth.as_f64(inp["g"]) if "g" in inp else None

    def step():
        if "sum" in w.ops:
            oracle.gauss_sum(x, y, wt, w.tau, rows=rows)
        if "lse" in w.ops:
            oracle.gauss_lse(x, y, wt, w.tau, rows=rows)
        if "bwd" in w.ops:
            oracle.gauss_sum_bwd(x, y, wt, g, w.tau, rows=rows, wrows=rows % w.N)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    pairs = w.B * len(rows) * w.N * (("sum" in w.ops or "bwd" in w.ops) + ("lse" in w.ops))
    value = pairs / dt / 1e9
    line = {"impl": "reference", "metric": "Gaussian kernel-sum pairs/sec (G pairs/s)",
            "value": value, "unit": "G pairs/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "M": w.M, "N": w.N, "D": w.D, "C": w.C,
                       "tau": w.tau, "ops": list(w.ops)},
            "cpu_baseline": {"kind": "oracle", "cores": base["cores"], "value": value,
                             "unit": "G pairs/s", "sample": base["sample"] + " per step"},
            "e2e": {"value": value, "unit": "G pairs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def main():
    args = parse()
    w = synth.BY_NAME[args.workload]
    if args.impl == "reference":
        return reference_arm(args, w)
    rank, world, local, pg = dist_init(args.gpus, need_group=args.sharded)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    import pairwise_reductions_b200 as gs
    dev = torch.device("cuda", local)
    if args.sharded:   # one problem: the workload's own seed on every rank, then this rank's slice
        inp = shard_of(synth.make_inputs(w), rank, world)
    else:              # independent problems: a seed per rank
        inp = synth.make_inputs(w, seed=(1000 + w.wid + 7919 * rank) if rank else None)
    d = {k: inp[k].to(dev) for k in ("x", "y", "w", "g") if k in inp}
    d["tau"] = inp["tau"]
    outs = {"sum": torch.empty(w.B, w.M, w.C, device=dev), "lse": torch.empty(w.B, w.M, w.C, device=dev)}
    if "bwd" in w.ops:
        outs["saved"] = torch.empty(w.B, w.M, w.C * (1 + w.D), device=dev)
        outs["gx"] = torch.empty(w.B, w.M, w.D, device=dev)
        outs["gw"] = torch.empty(w.B, w.N, w.C, device=dev)
    ws_bytes = max(gs.workspace_bytes(op, w.B, w.M, w.N, w.D, w.C, d["x"].dtype)
                   for op, name in ((gs.GS_OP_SUM, "sum"), (gs.GS_OP_LSE, "lse"), (gs.GS_OP_SUM_BWD, "bwd"),
                                    (gs.GS_OP_SUM_FWD_BWD, "bwd"))
                   if name in w.ops)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    counts = None
    if args.sharded:
        from pairwise_reductions_b200 import sharded
        counts = (sharded.shard_counts(d["x"].shape[1], dev), sharded.shard_counts(d["y"].shape[1], dev))
    run = sharded_step_fn(w, d, counts) if args.sharded else step_fn(gs, w, d, ws, outs, args.two_call)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    for _ in range(max(args.warmup, 3)):
        run()
    torch.cuda.synchronize()
    n_launch, kernel_names = (None, []) if args.no_launch_count else launches_per_step(gs, run)
    if gs.last_device_error() != 0:
        raise SystemExit("device error word set during warm-up")
    two_part = (not args.sharded) and "sum" in w.ops and "bwd" in w.ops and args.two_call
    # The timed steps replay one step captured in a CUDA graph: the same kernels
    # on the same buffers, without the host's launch gaps between them (which
    # matter at tens of microseconds a step).
    graph, graph_note = None, "host launches"
    if not args.no_graph and not args.sharded and not two_part:
        try:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                run()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            with torch.cuda.graph(g):
                run()
            torch.cuda.synchronize()
            graph, graph_note = g, "one step captured in a CUDA graph, replayed each timed step"
        except Exception as exc:   # capture unsupported here: time host launches
            graph, graph_note = None, f"host launches (graph capture failed: {type(exc).__name__})"

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)] if two_part else None
    clk_path = (args.clock_log.replace(".csv", f"_rank{rank}.csv") if args.clock_log
                else os.path.join(tempfile.gettempdir(), f"gs_clocks_{rank}.csv"))
    clk = ClockSampler(local, clk_path)
    barrier(pg)
    torch.cuda.synchronize()
    with clk:
        time.sleep(0.3)
        for k in range(args.steps):
            flush.fill_(float(k))
            starts[k].record(stream)
            if two_part:
                run(mids[k])
            elif graph is not None:
                graph.replay()
            else:
                run()
            ends[k].record(stream)
        torch.cuda.synchronize()
        time.sleep(0.2)
    barrier(pg)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    parts = None
    if two_part:
        # forward (keeping the x-gradient sums) and backward, each against B M N pairs
        f_ms = statistics.median(s.elapsed_time(m) for s, m in zip(starts, mids))
        b_ms = statistics.median(m.elapsed_time(e) for m, e in zip(mids, ends))
        parts = {"fwd_saved_ms": f_ms, "bwd_saved_ms": b_ms,
                 "fwd_g_pairs_s": w.pairs / (f_ms * 1e-3) / 1e9,
                 "bwd_g_pairs_s": w.pairs / (b_ms * 1e-3) / 1e9}
    total_ms = max_over_ranks(sum(step_ms), pg, dev)
    ms_per_step = total_ms / args.steps
    evals = pairs_per_step(w)   # one problem's pairs per step
    kevals = kernel_evals_per_step(w, args.two_call or args.sharded)
    jobs = 1 if args.sharded else world   # problems the whole job solves per step
    value = evals * jobs * args.steps / (total_ms * 1e-3) / 1e9
    if gs.last_device_error() != 0:
        raise SystemExit("device error word set during the timed loop")

    # ---- end to end through the public API: pinned host inputs -> device -> result -> host
    hx = {k: inp[k].pin_memory() for k in ("x", "y", "w", "g") if k in inp}
    # the step's results read back: the sum (or the log-sum-exp), and for the
    # one-call forward + backward step its two gradients too
    res_keys = ["lse" if "lse" in w.ops and "sum" not in w.ops else "sum"]
    if "bwd" in w.ops and not args.two_call and not args.sharded:
        res_keys += ["gx", "gw"]
    hres = {k: torch.empty(outs[k].shape).pin_memory() for k in res_keys[1:]}
    hres[res_keys[0]] = torch.empty(w.B, inp["x"].shape[1], w.C).pin_memory()   # this rank's rows
    hout = hres[res_keys[0]]
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = sum(t.numel() * t.element_size() for t in hres.values())
    e_s = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)

    def e2e_step():
        dd = {k: t.to(dev, non_blocking=True) for k, t in hx.items()}
        dd["tau"] = inp["tau"]
        if args.sharded:
            sharded_step_fn(w, dd, counts)()
            hout.copy_(dd["out_lse" if "lse" in w.ops and "sum" not in w.ops else "out_sum"],
                       non_blocking=True)
        else:
            step_fn(gs, w, dd, ws, outs, args.two_call)()
            for k in res_keys:
                hres[k].copy_(outs[k], non_blocking=True)

    # Independent problems: two lanes, each with its own stream, device buffers,
    # workspace and pinned result buffer; step k runs on lane k % 2, so the
    # copies of one step overlap the pair work of the other (every step still
    # copies its own inputs in and its result out inside the timed region).
    lanes = []
    if not args.sharded:
        for _ in range(2):
            ln = {"stream": torch.cuda.Stream(device=dev),
                  "d": {k: torch.empty_like(t, device=dev) for k, t in hx.items()},
                  "outs": {k: torch.empty_like(v) for k, v in outs.items()},
                  "ws": torch.empty_like(ws),
                  "hres": {k: torch.empty_like(t).pin_memory() for k, t in hres.items()}}
            ln["d"]["tau"] = inp["tau"]
            lanes.append(ln)

    def e2e_lane_step(ln):
        with torch.cuda.stream(ln["stream"]):
            for k, t in hx.items():
                ln["d"][k].copy_(t, non_blocking=True)
            step_fn(gs, w, ln["d"], ln["ws"], ln["outs"], args.two_call)()
            for k in res_keys:
                ln["hres"][k].copy_(ln["outs"][k], non_blocking=True)

    e2e_ms, e2e_value = None, None
    if args.e2e_steps > 0:
        for k in range(2):
            e2e_step() if args.sharded else e2e_lane_step(lanes[k % 2])
        torch.cuda.synchronize()
        barrier(pg)
        e_s.record(stream)
        for ln in lanes:
            ln["stream"].wait_event(e_s)
        for k in range(args.e2e_steps):
            e2e_step() if args.sharded else e2e_lane_step(lanes[k % 2])
        for ln in lanes:
            stream.wait_stream(ln["stream"])
        e_e.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e_s.elapsed_time(e_e), pg, dev) / args.e2e_steps
        e2e_value = evals * jobs / (e2e_ms * 1e-3) / 1e9
    # One call at a time on one stream: copies in, the step, the result out,
    # each step between its own start and end events (the latency one call sees).
    single = None
    if args.e2e_single_steps > 0 and not args.sharded:
        ln = lanes[0]
        e2e_lane_step(ln)
        torch.cuda.synchronize()
        barrier(pg)
        one = []
        for _ in range(args.e2e_single_steps):
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(ln["stream"])
            e2e_lane_step(ln)
            z.record(ln["stream"])
            ln["stream"].synchronize()
            one.append(a.elapsed_time(z))
        single_ms = max_over_ranks(statistics.median(one), pg, dev)
        single = {"value": evals * jobs / (single_ms * 1e-3) / 1e9, "ms_per_step": single_ms,
                  "steps": args.e2e_single_steps,
                  "pipelining": "none: one stream, each call finished before the next starts"}
    clocks = clk.summary()

    if rank == 0:
        props = torch.cuda.get_device_properties(dev)
        sms = props.multi_processor_count
        peaks = {}
        try:
            peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        except (OSError, ValueError):
            pass
        sm_max = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz") or 1965.0)
        peak = EX2_PER_CLK_PER_SM * sms * sm_max * 1e6 / 1e9
        # kernel evaluations (one MUFU ex2 each) per second on one GPU
        achieved = kevals * jobs / world / (ms_per_step * 1e-3) / 1e9
        traffic, dom = traffic_per_launch(w)
        roof = {"bound": "alu", "kernel": f"{dom}: one MUFU ex2 per kernel evaluation",
                "achieved": achieved, "peak": peak, "unit": "G kernel evaluations/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_basis": f"16 ex2/clk/SM x {sms} SMs x {sm_max:.0f} MHz (max SM clock)"}
        if clocks.get("sm_mhz"):
            roof["frac_at_measured_clock"] = achieved / (EX2_PER_CLK_PER_SM * sms * clocks["sm_mhz"] * 1e-3)
        # The binding resource: the tensor pipe where the step's MMA FLOPs need more time
        # at the measured dense bf16 / fp16 rate than its exponentials at the MUFU rate.
        tf = tensor_flops_per_step(w) * jobs / world
        t_peak = peaks.get("bf16_tflops")
        if tf and t_peak and tf / (t_peak * 1e12) > kevals * jobs / world / (peak * 1e9):
            t_ach = tf / (ms_per_step * 1e-3) / 1e12
            roof = {"bound": "tensor",
                    "kernel": f"{dom}: fp16 MMAs, {tf / (kevals * jobs / world):.0f} FLOP per pair",
                    "achieved": t_ach, "peak": t_peak, "unit": "TFLOP/s", "frac": t_ach / t_peak,
                    "traffic": traffic,
                    "peak_basis": "measured cuBLAS bf16 GEMM, burst (fp16 has the same rate)",
                    "frac_of_sustained": t_ach / peaks["bf16_tflops_sustained"]
                    if peaks.get("bf16_tflops_sustained") else None,
                    "alu": {"achieved": achieved, "peak": peak, "unit": "G kernel evaluations/s",
                            "frac": achieved / peak}}
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu, _ = oracle_sample(w, inp, args.cpu_seconds)
        pub = PUBLISHED.get(w.name)
        line = {"metric": "Gaussian kernel-sum pairs/sec (G pairs/s)", "value": value,
                "unit": "G pairs/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_per_step, "higher_is_better": True,
                "scaling": "strong" if args.sharded else "weak",
                "vs_baseline": (value / pub["value"]) if pub else None,
                "dtype": w.dtype, "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "M": w.M, "N": w.N, "D": w.D, "C": w.C,
                           "tau": w.tau, "ops": list(w.ops), "pairs_per_step": evals,
                           "kernel_evaluations_per_step": kevals,
                           "l2": "flushed by a 256 MiB write between timed steps",
                           "launch": graph_note,
                           "parallelism": (f"one problem sharded over {world} rank(s): rows and "
                                           f"sources split, sources all-gathered each step")
                           if args.sharded else f"independent problems, {world} rank(s)"},
                "roofline": roof, "cpu_baseline": cpu,
                "e2e": {"value": e2e_value, "unit": "G pairs/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                        "pipelining": "none (sharded)" if args.sharded else
                        "two streams: step k+1's copies overlap step k's pair work",
                        "single_call": single},
                "gpu_launches": (n_launch * args.steps) if n_launch is not None else None, "kernels": kernel_names,
                "clocks": clocks}
        if parts is not None:
            line["parts"] = parts   # rank 0's medians
        print(json.dumps(line), flush=True)
    graph = None   # released before the process group
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
