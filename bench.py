#!/usr/bin/env python
"""Benchmark of the fused LM-head projection + cross-entropy (forward + backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one forward and one backward of the whole path (projection GEMM with
the online-logsumexp epilogue, merge and loss, recompute GEMM with the gradient
epilogue, dW and dhidden GEMMs) over one batch of the seeded synthetic
workload, on inputs already resident in HBM.  The default workload is
N=4096 tokens (2 x 2048), H=4096, V=128256 (BF16 head N(0, 0.02), 5% of labels
ignored, loss summed and divided by the number of label tokens).

Under torchrun (N > 1) every rank runs its own replica of the workload on its
own GPU (weak scaling, no collective on the data path: the path computes one
loss per batch and has no exchange step of its own); timing takes the max over
ranks.  Rank 0 prints one JSON line.

--impl reference times the FP64 CPU oracle (the test oracle, as it stands) on
the host cores, on rank 0 only, each step a bounded token sample of the same
workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused linear-CE fwd+bwd tokens/sec on 1 B200; % of dense-BF16 tensor peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "n4096_h4096_v128256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic_per_launch.md")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--path", choices=["flce", "chunked_ce"], default="flce",
                    help="flce: the fused projection + CE (default); chunked_ce: cross entropy "
                         "on given logits [4096, 128256] BF16")
    ap.add_argument("--graph", action="store_true",
                    help="time flce.CapturedStep (forward + backward replayed from one CUDA "
                         "graph) instead of the eager calls; per-kernel figures are then not "
                         "available and the roofline covers the whole step")
    return ap.parse_args(argv)


# --------------------------------------------------------------------- helpers

def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_digest() -> str:
    """sha256 over the CUDA sources: ties committed ncu counters to the kernels they measured."""
    from lm_head_projection_flce_b200 import build as B
    h = hashlib.sha256()
    for p in B.sources():
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str, family: str) -> float | None:
    """DRAM bytes per launch of `family` from the committed ncu summary, if it was
    taken on the current kernel sources and this workload; else None."""
    try:
        text = open(PROFILE_TRAFFIC).read()
    except OSError:
        return None
    digest = kernel_source_digest()
    for line in text.splitlines():
        # | family | workload | source digest | dram bytes per launch | ...
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == family and cells[1] == workload and cells[2] == digest:
            try:
                return float(cells[3])
            except ValueError:
                return None
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.proc = None
        self.path = None
        self.uuid = gpu_uuid

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="flce_clocks_", suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100", "-f", self.path]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        try:
            rows = open(self.path).read().splitlines()
        finally:
            os.unlink(self.path)
        return self.summarize(rows)

    @staticmethod
    def summarize(rows: list[str]) -> dict:
        """Median SM clock, max clock and the throttle reasons seen in the CSV rows."""
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in rows:
            c = [x.strip() for x in row.split(",")]
            if len(c) < 9:
                continue
            try:
                sm.append(float(c[1]))
                smax.append(float(c[2]))
                power.append(float(c[3]))
            except ValueError:
                continue
            for name, val in zip(names, c[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power) if power else None, "samples": len(sm),
                "reasons": sorted(reasons)}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def workload_config(w, parallelism: str) -> dict:
    return {
        "workload": w.name, "n_tokens": w.n_tokens, "batch": w.batch, "seq": w.seq,
        "hidden": w.hidden, "vocab": w.vocab, "padded_vocab": w.padded_vocab,
        "head_dtype": w.w_dtype, "softcap": w.softcap, "ignore_frac": w.ignore_frac,
        "labels": w.label_dist,
        "reduction": w.reduction + ("/num_label_tokens" if w.normalize_by_label_tokens else ""),
        "parallelism": parallelism,
        "l2": (f"inputs larger than L2: the {w.padded_vocab * w.hidden * (2 if w.w_dtype == 'bf16' else 4) / 1e9:.2f} GB "
               "head is streamed from HBM every step (L2 is 126 MB)"),
    }


def reduce_max(x: float, device) -> float:
    """Max of a per-rank float over the default process group (identity when alone)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(tokens_per_rank: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's device time."""
    return tokens_per_rank * steps * world / (ms_max / 1e3)


# ------------------------------------------------------------------ CPU oracle

def oracle_inputs(d: dict):
    hidden = d["hidden"].double().numpy()
    w = d["weight"]
    weight = w.numpy() if w.dtype.is_floating_point and w.element_size() == 4 else w.double().numpy()
    return hidden, weight, d["labels"].numpy()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_step(O, w, hidden, weight, labels, rows, num_label_tokens):
    """One oracle forward + backward over the token rows `rows` (full V and H)."""
    kw = dict(ignore_index=-100, softcap=w.softcap, unpadded_vocab=w.vocab, reduction=w.reduction,
              num_label_tokens=num_label_tokens)
    O.forward(hidden[rows], weight, labels[rows], **kw)
    O.backward(hidden[rows], weight, labels[rows], **kw)


def cpu_baseline(w, d, target_s: float = 15.0, max_tokens: int = 4096) -> dict:
    """Time the oracle on a seeded token sample of the workload (about `target_s` of CPU work)."""
    import numpy as np
    from oracle import flce_oracle as O
    hidden, weight, labels = oracle_inputs(d)
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    rng = np.random.default_rng(7)
    # Grow the sample (x4) until one oracle pass takes about target_s / 4 or more;
    # the oracle has a fixed per-call cost (the full [Vp, H] dW), so probe sizes grow.
    s = min(16, w.n_tokens)
    while True:
        rows = rng.choice(w.n_tokens, size=s, replace=False)
        t0 = time.perf_counter()
        oracle_step(O, w, hidden, weight, labels, rows, nlt)
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or s >= min(max_tokens, w.n_tokens):
            break
        s = min(4 * s, max_tokens, w.n_tokens)
    # The timed sample: scaled so that one oracle pass takes about target_s.
    s = int(min(max_tokens, w.n_tokens, max(s, s * target_s / max(dt, 1e-3))))
    rows = rng.choice(w.n_tokens, size=s, replace=False)
    t0 = time.perf_counter()
    oracle_step(O, w, hidden, weight, labels, rows, nlt)
    dt = time.perf_counter() - t0
    return {"value": s / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{s} seeded tokens of {w.name} through the FP64 oracle's full forward + "
                       f"backward (lse over all {w.vocab} rows, their dhidden rows and their "
                       f"contribution to all of dW), {dt:.1f} s; numpy/OpenBLAS FP64")}


def run_reference(args, w) -> int:
    """--impl reference: the oracle on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    from lm_head_projection_flce_b200 import workloads as W
    from oracle import flce_oracle as O
    d = W.generate(w)
    hidden, weight, labels = oracle_inputs(d)
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    warmup = max(args.warmup, 3)
    rng = np.random.default_rng(11)
    t0 = time.perf_counter()
    oracle_step(O, w, hidden, weight, labels, rng.choice(w.n_tokens, 4, replace=False), nlt)
    t4 = time.perf_counter() - t0
    budget = 150.0 / (args.steps + warmup)            # seconds per step for the whole run
    s = int(max(1, min(256, w.n_tokens, budget / max(t4, 1e-3) * 4)))
    for _ in range(warmup):
        oracle_step(O, w, hidden, weight, labels, rng.choice(w.n_tokens, s, replace=False), nlt)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(O, w, hidden, weight, labels, rng.choice(w.n_tokens, s, replace=False), nlt)
    dt = time.perf_counter() - t0
    value = s * args.steps / dt
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, "host cores (rank 0 only)"),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": (f"each step: {s} seeded tokens of {w.name} through the FP64 "
                                    "oracle's full forward + backward")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU path

def run_ours(args, w) -> int:
    import torch
    import torch.distributed as dist

    from lm_head_projection_flce_b200 import flce
    from lm_head_projection_flce_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (sm_100a)")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, dev)

    from lm_head_projection_flce_b200 import build as B
    B.build()                               # no-op when the in-tree library matches its sources
    flce.load_library()
    d = W.generate(w)                       # seeded on the CPU: the same batch on every rank
    hid = d["hidden"].to(dev)
    wt = d["weight"].to(dev)
    lab = d["labels"].to(dev)
    n, h, vp, v = w.n_tokens, w.hidden, w.padded_vocab, w.vocab
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    ws = torch.empty(flce.workspace_size(n, h, vp, v, wt.dtype), dtype=torch.uint8, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(n, dtype=torch.float32, device=dev)
    dh = torch.empty_like(hid)
    dw = torch.empty_like(wt)
    grad = torch.ones(1, dtype=torch.float32, device=dev)
    kw = dict(softcap=w.softcap, unpadded_vocab=v, reduction=w.reduction, num_label_tokens=nlt,
              workspace=ws)

    def step(h_in=hid, l_in=lab):
        flce.forward(h_in, wt, l_in, loss=loss, lse=lse, **kw)
        flce.backward(h_in, wt, l_in, lse, grad, dhidden=dh, dweight=dw, **kw)

    captured = None
    if args.graph:
        l0 = flce.launch_count()
        captured = flce.CapturedStep(hid, wt, lab, softcap=w.softcap, unpadded_vocab=v,
                                     reduction=w.reduction, num_label_tokens=nlt)
        graph_launches = (flce.launch_count() - l0) // 2  # the eager set-up step + the capture
        loss = captured.loss

        def step(h_in=None, l_in=None):  # noqa: F811 - the graph replaces the eager calls
            if h_in is not None:
                captured.set_inputs(h_in, l_in)
            captured.replay()

    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    status = flce.get_error(dev)
    if status != flce.FLCE_OK:
        raise RuntimeError(f"device error during warm-up: {flce.STATUS[status]}")

    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    stream = torch.cuda.current_stream(dev)

    def timed_region(profile: bool):
        sampler = ClockSampler(uuid)
        sampler.start()
        barrier()
        torch.cuda.synchronize(dev)
        if profile:
            flce.profile_start()
        l0 = flce.launch_count()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        launches = flce.launch_count() - l0
        stats = flce.profile_stop() if profile else {}
        clocks = sampler.stop()
        return e0.elapsed_time(e1), launches, stats, clocks

    # The headline pass runs without per-launch events (a few microseconds per
    # launch, which shows on small workloads); the per-kernel figures of the
    # roofline come from a second pass of the same steps with the events on.
    ms, launches, _, clocks = timed_region(False)
    remeasured = False
    # Re-measure once if any rank saw a hardware or thermal slowdown; the
    # decision is collective so every rank takes the same barriers.
    bad = 1.0 if BAD_REASONS & set(clocks.get("reasons", [])) else 0.0
    if max_over_ranks(bad) > 0:
        ms, launches, _, clocks = timed_region(False)
        remeasured = True
    stats = timed_region(True)[2] if captured is None else {}
    if captured is not None:  # replays enqueue no library call: count the graph's kernels
        launches = graph_launches * args.steps
    ms_max = max_over_ranks(ms)
    if flce.get_error(dev) != flce.FLCE_OK:
        raise RuntimeError("device error word set during the timed region")

    # ---- end to end: pinned host inputs -> device, fwd + bwd, loss -> host, every step.
    # Step k+1's inputs are copied on a second stream into the other of two
    # device buffers while step k computes; every copy is inside the timed
    # region (the copy stream starts after e0, the last step waits for its copy).
    h_host = d["hidden"].pin_memory()
    l_host = d["labels"].pin_memory()
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()
    copy_stream = torch.cuda.Stream(dev)
    bufs = [(torch.empty_like(hid), torch.empty_like(lab)) for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def stage(k):
        b = k % 2
        copy_stream.wait_event(consumed[b])     # the step that last read buffer b is done
        with torch.cuda.stream(copy_stream):
            bufs[b][0].copy_(h_host, non_blocking=True)
            bufs[b][1].copy_(l_host, non_blocking=True)
        copied[b].record(copy_stream)

    def e2e_run(steps, start_event=None):
        if start_event is not None:
            copy_stream.wait_event(start_event)
        stage(0)
        for k in range(steps):
            if k + 1 < steps:
                stage(k + 1)
            b = k % 2
            stream.wait_event(copied[b])
            step(*bufs[b])
            consumed[b].record(stream)
            loss_host.copy_(loss, non_blocking=True)

    e2e_run(2)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps, e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))

    value = aggregate_throughput(n, args.steps, world, ms_max)
    e2e_value = aggregate_throughput(n, args.steps, world, e2e_ms)

    peaks, peak_src = load_peaks()
    gemms = {k: s for k, s in stats.items() if s["flops"] > 0}
    if captured is None:
        dom_name = max(gemms, key=lambda k: gemms[k]["total_ms"])
        dom = gemms[dom_name]
    else:  # graph replays carry no per-launch events: the whole step is the unit
        dom_name = "whole step (CUDA graph replay)"
        dom = {"flops": w.flops_fwd_bwd * args.steps, "total_ms": ms_max,
               "launches": graph_launches * args.steps}
    achieved = dom["flops"] / (dom["total_ms"] / 1e3) / 1e12
    # The kernels are timed inside a seconds-long continuous run (clocks settle
    # under the power cap), so the sustained GEMM figure is the denominator;
    # the burst figure is reported beside it.
    peak_burst = float(peaks["bf16_tflops"])
    peak = float(peaks.get("bf16_tflops_sustained", peak_burst))
    per_step_launches = dom["launches"] / args.steps
    traffic = committed_traffic(w.name, dom_name)
    kernels = {k: {"launches_per_step": s["launches"] / args.steps,
                   "ms_per_step": s["total_ms"] / args.steps,
                   **({"tflops": s["flops"] / (s["total_ms"] / 1e3) / 1e12} if s["flops"] > 0 else
                      {"gbs": s["bytes"] / (s["total_ms"] / 1e3) / 1e9 if s["total_ms"] > 0 else None})}
               for k, s in sorted(stats.items())}
    path_flops = w.flops_fwd_bwd * args.steps * world

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(w, f"replicas x{world} (one independent batch per GPU)"),
                       **({"cuda_graph": True} if captured is not None else {})},
            "roofline": {
                "bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + write.sum)",
                "flops_per_launch": dom["flops"] / dom["launches"],
                "launches_per_step": per_step_launches,
                "peak_source": f"{peak_src} bf16_tflops_sustained (cuBLAS, seconds-long loop)",
                "peak_burst": peak_burst, "frac_of_burst": achieved / peak_burst,
                "whole_path_tflops": path_flops / (ms_max / 1e3) / 1e12 / world,
                "whole_path_frac": path_flops / (ms_max / 1e3) / 1e12 / world / peak,
                "whole_path_frac_of_burst": path_flops / (ms_max / 1e3) / 1e12 / world / peak_burst,
            },
            "kernels": kernels,
            "kernel_timing": ("per-launch CUDA events in a second pass of the same steps"
                              if captured is None else "none inside a CUDA graph"),
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": hid.numel() * hid.element_size() + lab.numel() * 8,
                    "d2h_bytes_per_step": 4,
                    "api": "lm_head_projection_flce_b200.flce.forward/backward (C ABI via ctypes)",
                    "overlap": "step k+1's H2D copy on a second stream during step k"},
            "gpu_launches": launches,
            "clocks": {**clocks, "remeasured": remeasured},
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, d)
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()
    return 0


def run_chunked_ce(args) -> int:
    """Cross entropy on given logits: forward + backward per step (HBM-bound)."""
    import torch

    from lm_head_projection_flce_b200 import flce
    from lm_head_projection_flce_b200 import workloads as W

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (sm_100a)")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    from lm_head_projection_flce_b200 import build as B
    B.build()
    flce.load_library()
    w = W.CE_LOGITS
    d = W.generate_logits(w)
    z = d["logits"].to(dev)
    lab = d["labels"].to(dev)
    n, v = z.shape
    nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
    ws = torch.empty(int(flce.load_library().flce_ce_workspace_size(n)), dtype=torch.uint8,
                     device=dev)
    dz = torch.empty_like(z)
    grad = torch.ones(1, device=dev)

    def step(z_in=z, l_in=lab):
        loss, lse = flce.ce_forward(z_in, l_in, reduction=w.reduction, num_label_tokens=nlt,
                                    workspace=ws)
        flce.ce_backward(z_in, l_in, lse, grad, reduction=w.reduction, num_label_tokens=nlt,
                         dlogits=dz, workspace=ws)
        return loss

    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    def timed(profile: bool):
        torch.cuda.synchronize(dev)
        if profile:
            flce.profile_start()
        l0 = flce.launch_count()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        launches = flce.launch_count() - l0
        stats = flce.profile_stop() if profile else None
        return e0.elapsed_time(e1), launches, stats

    # The steps here are ~0.5 ms, so the per-launch events of the kernel
    # profile would add a few percent: the step time comes from a pass
    # without them, the per-kernel figures from a second, profiled pass.
    sampler = ClockSampler(uuid)
    sampler.start()
    ms, launches, _ = timed(False)
    _, _, stats = timed(True)
    clocks = sampler.stop()
    if flce.get_error(dev) != flce.FLCE_OK:
        raise RuntimeError("device error word set during the timed region")
    peaks, peak_src = load_peaks()
    hbm = [k for k, st in stats.items() if st["bytes"] > 0 and k.startswith("ce_logits")]
    dom_name = max(hbm, key=lambda k: stats[k]["total_ms"])
    dom = stats[dom_name]
    achieved = dom["bytes"] / (dom["total_ms"] / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    line = {
        "metric": "cross entropy on given logits, fwd+bwd tokens/sec on 1 B200",
        "value": n * args.steps / (ms / 1e3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "n_tokens": n, "vocab": v, "logits_dtype": w.dtype,
                   "logits_sigma": w.sigma, "ignore_frac": w.ignore_frac,
                   "reduction": "sum/num_label_tokens",
                   "l2": "inputs larger than L2: 1.05 GB of logits read twice and 1.05 GB of "
                         "gradient written every step"},
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "traffic": committed_traffic(w.name, dom_name),
                     "bytes_per_launch": dom["bytes"] / dom["launches"],
                     "peak_source": f"{peak_src} hbm_gbs (copy read+write)"},
        "kernels": {k: {"launches_per_step": st["launches"] / args.steps,
                        "ms_per_step": st["total_ms"] / args.steps,
                        "gbs": st["bytes"] / (st["total_ms"] / 1e3) / 1e9 if st["total_ms"] > 0 else None}
                    for k, st in sorted(stats.items())},
        "kernel_timing": "per-launch CUDA events in a second pass of the same steps",
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    if args.path == "chunked_ce":
        return run_chunked_ce(args)
    from lm_head_projection_flce_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
