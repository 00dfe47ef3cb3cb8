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
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic_per_launch.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the short timed passes of the other large workloads and of cross "
                         "entropy on given logits (one GPU only) under 'extra_workloads'")
    ap.add_argument("--fused-head-cast", action="store_true",
                    help="with an FP32 head, round it to BF16 inside the GEMMs "
                         "(FLCE_FUSED_HEAD_CAST) instead of casting it into a copy")
    ap.add_argument("--extra-steps", type=int, default=5,
                    help="timed steps of each extra workload (at least 5)")
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
    """DRAM bytes per launch of `family` on `workload` from the committed ncu
    record (profiles/dram_traffic_per_launch.json), if it was taken on the
    current kernel sources; else None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            records = json.load(f)["records"]
    except (OSError, ValueError, KeyError, TypeError):
        return None
    digest = kernel_source_digest()
    for r in records:
        if (r.get("family") == family and r.get("workload") == workload
                and r.get("source_digest") == digest):
            try:
                return float(r["bytes_per_launch"])
            except (KeyError, TypeError, ValueError):
                return None
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "timestamp")

    def __init__(self, gpu_uuid: str | None):
        self.proc = None
        self.path = None
        self.uuid = gpu_uuid
        self.window = None

    def mark(self, begin: float, end: float):
        """Host wall-clock bounds of the timed region: only samples taken inside it
        (plus one sampling period after it) are summarised."""
        self.window = (begin, end + 0.1)

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
        return self.summarize(rows, self.window)

    @staticmethod
    def sample_time(field: str) -> float | None:
        """nvidia-smi's timestamp (local time, 'YYYY/MM/DD HH:MM:SS.mmm') as epoch seconds."""
        try:
            return datetime.datetime.strptime(field.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    @staticmethod
    def summarize(rows: list[str], window: tuple | None = None) -> dict:
        """Median SM clock, max clock and the throttle reasons seen in the CSV rows
        (only rows whose timestamp lies in `window`, when one is given and some do)."""
        if window is not None:
            inside = []
            for row in rows:
                c = [x.strip() for x in row.split(",")]
                t = ClockSampler.sample_time(c[9]) if len(c) >= 10 else None
                if t is not None and window[0] <= t <= window[1]:
                    inside.append(row)
            if inside:
                rows = inside
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
    # The timed sample: scaled so that one oracle pass takes about target_s (the
    # last probe already is that pass when the size does not change).
    s_next = int(min(max_tokens, w.n_tokens, max(s, s * target_s / max(dt, 1e-3))))
    if s_next != s:
        s = s_next
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

def tensor_roofline(stats: dict, peaks: dict, peak_src: str, workload: str,
                    whole_path_flops: float, whole_path_ms: float) -> dict:
    """Roofline of the dominant contraction (the kernel family with the most device
    time): algorithmic FLOPs / its CUDA-event time against the measured dense-BF16
    peak.  The denominator is the burst cuBLAS figure -- the bench's timed
    regions are a fraction of a second to a few seconds, the regime that figure
    was taken in; the sustained (power-capped, seconds-long loop) figure is
    reported beside it.  A fraction above 1 means the timed kernel did not do the
    work it claims, so it is refused (frac null) rather than reported."""
    gemms = {k: v for k, v in stats.items() if v["flops"] > 0}
    name = max(gemms, key=lambda k: gemms[k]["total_ms"])
    dom = gemms[name]
    achieved = dom["flops"] / (dom["total_ms"] / 1e3) / 1e12
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    whole = whole_path_flops / (whole_path_ms / 1e3) / 1e12
    out = {
        "bound": "tensor", "kernel": name, "achieved": achieved, "peak": burst,
        "unit": "TFLOP/s", "frac": achieved / burst,
        "traffic": committed_traffic(workload, name),
        "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + write.sum)",
        "flops_per_launch": dom["flops"] / dom["launches"],
        "launches": dom["launches"],
        "peak_source": f"{peak_src} bf16_tflops (cuBLAS dense BF16, burst)",
        "peak_sustained": sustained, "frac_of_sustained": achieved / sustained,
        "whole_path_tflops": whole, "whole_path_frac": whole / burst,
    }
    if out["frac"] > 1.0 or out["whole_path_frac"] > 1.0:
        out["frac_refused"] = (f"{out['frac']:.3f} / {out['whole_path_frac']:.3f} of the burst "
                               "peak: above 1, so the timing does not cover the work claimed")
        out["frac"] = None
        out["whole_path_frac"] = None
    return out


def hbm_roofline(stats: dict, peaks: dict, peak_src: str, workload: str, prefix: str) -> dict:
    """Roofline of the dominant single-pass HBM kernel: algorithmic bytes / time
    against the measured copy bandwidth (refused above 1, as for the GEMMs)."""
    hbm = {k: v for k, v in stats.items() if v["bytes"] > 0 and k.startswith(prefix)}
    name = max(hbm, key=lambda k: hbm[k]["total_ms"])
    dom = hbm[name]
    achieved = dom["bytes"] / (dom["total_ms"] / 1e3) / 1e9
    peak = float(peaks["hbm_gbs"])
    out = {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": peak, "unit": "GB/s",
           "frac": achieved / peak, "traffic": committed_traffic(workload, name),
           "bytes_per_launch": dom["bytes"] / dom["launches"],
           "peak_source": f"{peak_src} hbm_gbs (copy read+write)"}
    if out["frac"] > 1.0:
        out["frac_refused"] = f"{out['frac']:.3f} of the copy bandwidth: above 1"
        out["frac"] = None
    return out


def cublas_same_run(dev, stream, seconds: float) -> dict:
    """cuBLAS (torch.matmul) dense BF16 8192^3 timed right after our timed region
    for about as long, so it runs in the same power / clock regime: a measuring
    stick for the roofline (the contract's peak stays the measured burst figure)."""
    import torch
    a = torch.randn(8192, 8192, device=dev, dtype=torch.bfloat16)
    b = torch.randn(8192, 8192, device=dev, dtype=torch.bfloat16)
    for _ in range(3):
        torch.matmul(a, b)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    torch.matmul(a, b)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    reps = int(min(2000, max(10, seconds / max(e0.elapsed_time(e1) / 1e3, 1e-5))))
    e0.record(stream)
    for _ in range(reps):
        torch.matmul(a, b)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    del a, b
    return {"tflops": 2.0 * 8192 ** 3 / (ms / 1e3) / 1e12, "ms_per_gemm": ms, "gemms": reps,
            "what": "torch.matmul BF16 8192x8192x8192 (cuBLAS), timed right after the headline "
                    "pass for about as long"}


def kernel_table(stats: dict, steps: int) -> dict:
    return {k: {"launches_per_step": st["launches"] / steps,
                "ms_per_step": st["total_ms"] / steps,
                **({"tflops": st["flops"] / (st["total_ms"] / 1e3) / 1e12} if st["flops"] > 0 else
                   {"gbs": st["bytes"] / (st["total_ms"] / 1e3) / 1e9 if st["total_ms"] > 0
                    else None})}
            for k, st in sorted(stats.items())}


class Timer:
    """Device timing of `steps` calls of `step` on `stream`: CUDA events on the
    launching stream around the whole region (barrier + synchronize on both
    sides) and between steps, the library's launch count, optionally its
    per-launch events, and nvidia-smi clock samples taken meanwhile."""

    def __init__(self, dev, stream, uuid, barrier=lambda: None):
        self.dev, self.stream, self.uuid, self.barrier = dev, stream, uuid, barrier

    def run(self, step, steps: int, profile: bool = False):
        import torch
        from lm_head_projection_flce_b200 import flce
        sampler = ClockSampler(self.uuid)
        sampler.start()
        self.barrier()
        torch.cuda.synchronize(self.dev)
        if profile:
            flce.profile_start()
        l0 = flce.launch_count()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        t_begin = time.time()
        ev[0].record(self.stream)
        for k in range(steps):
            step()
            ev[k + 1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        sampler.mark(t_begin, time.time())
        self.barrier()
        launches = flce.launch_count() - l0
        stats = flce.profile_stop() if profile else {}
        clocks = sampler.stop()
        per_step = [ev[k].elapsed_time(ev[k + 1]) for k in range(steps)]
        return {"ms": ev[0].elapsed_time(ev[steps]), "per_step": per_step,
                "launches": launches, "stats": stats, "clocks": clocks}


class FlceRun:
    """One workload's inputs, outputs and workspace on the device, and its step:
    forward + backward through the binding, the backward reusing the forward's
    BF16 copy of an FP32 head (same workspace, head unchanged in between)."""

    def __init__(self, w, dev, graph: bool = False):
        import torch
        from lm_head_projection_flce_b200 import flce
        from lm_head_projection_flce_b200 import workloads as W
        self.w = w
        self.data = W.generate(w)           # seeded on the CPU: the same batch on every rank
        d = self.data
        self.hid = d["hidden"].to(dev)
        self.wt = d["weight"].to(dev)
        self.lab = d["labels"].to(dev)
        n, h, vp, v = w.n_tokens, w.hidden, w.padded_vocab, w.vocab
        self.nlt = d["num_label_tokens"] if w.normalize_by_label_tokens else None
        self.ws = torch.empty(flce.workspace_size(n, h, vp, v, self.wt.dtype), dtype=torch.uint8,
                              device=dev)
        self.loss = torch.empty(1, dtype=torch.float32, device=dev)
        self.lse = torch.empty(n, dtype=torch.float32, device=dev)
        self.dh = torch.empty_like(self.hid)
        self.dw = torch.empty_like(self.wt)
        self.grad = torch.ones(1, dtype=torch.float32, device=dev)
        self.kw = dict(softcap=w.softcap, unpadded_vocab=v, reduction=w.reduction,
                       num_label_tokens=self.nlt, workspace=self.ws)
        self.reuse = self.wt.dtype == torch.float32
        self.fused_cast = False
        self.label = w.name  # names the committed traffic record this run's kernels match
        self.captured = None
        self.graph_launches = 0
        if graph:
            l0 = flce.launch_count()
            self.captured = flce.CapturedStep(self.hid, self.wt, self.lab, softcap=w.softcap,
                                              unpadded_vocab=v, reduction=w.reduction,
                                              num_label_tokens=self.nlt)
            self.graph_launches = (flce.launch_count() - l0) // 2  # eager set-up + capture
            self.loss = self.captured.loss

    def use_fused_head_cast(self, dev):
        """Switch an FP32-head run to FLCE_FUSED_HEAD_CAST: the GEMMs round the
        head in the kernel, with the smaller workspace that has no BF16 copy."""
        import torch
        from lm_head_projection_flce_b200 import flce
        w = self.w
        self.ws = None
        self.ws = torch.empty(flce.workspace_size(w.n_tokens, w.hidden, w.padded_vocab, w.vocab,
                                                  self.wt.dtype, fused_head_cast=True),
                              dtype=torch.uint8, device=dev)
        self.kw["workspace"] = self.ws
        self.reuse = False
        self.fused_cast = True
        self.label = w.name + "/fused_head_cast"

    def step(self, h_in=None, l_in=None):
        from lm_head_projection_flce_b200 import flce
        if self.captured is not None:
            if h_in is not None:
                self.captured.set_inputs(h_in, l_in)
            self.captured.replay()
            return
        h_in = self.hid if h_in is None else h_in
        l_in = self.lab if l_in is None else l_in
        flce.forward(h_in, self.wt, l_in, loss=self.loss, lse=self.lse,
                     fused_head_cast=self.fused_cast, **self.kw)
        flce.backward(h_in, self.wt, l_in, self.lse, self.grad, dhidden=self.dh, dweight=self.dw,
                      reuse_head_copy=self.reuse, fused_head_cast=self.fused_cast, **self.kw)


def measure_flce(run: "FlceRun", timer: "Timer", steps: int, warmup: int, world: int,
                 max_over_ranks, peaks, peak_src, after_headline=None) -> dict:
    """Warm-up, the headline pass (no per-launch events), a re-measure if any
    rank saw a hardware/thermal slowdown, `after_headline(headline)` (the
    end-to-end pass and the same-run cuBLAS reference, so they run in the
    headline's power regime), then a profiled pass for the kernel table."""
    import torch
    from lm_head_projection_flce_b200 import flce
    dev = timer.dev
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize(dev)
    status = flce.get_error(dev)
    if status != flce.FLCE_OK:
        raise RuntimeError(f"device error during warm-up: {flce.STATUS[status]}")
    head = timer.run(run.step, steps)
    remeasured = False
    # The decision is collective so every rank takes the same barriers.
    bad = 1.0 if BAD_REASONS & set(head["clocks"].get("reasons", [])) else 0.0
    if max_over_ranks(bad) > 0:
        head = timer.run(run.step, steps)
        remeasured = True
    between = after_headline(head) if after_headline is not None else None
    prof = timer.run(run.step, steps, profile=True) if run.captured is None else None
    if flce.get_error(dev) != flce.FLCE_OK:
        raise RuntimeError("device error word set during the timed region")
    ms_max = max_over_ranks(head["ms"])
    w = run.w
    path_flops = w.flops_fwd_bwd * steps
    if prof is not None:
        roof = tensor_roofline(prof["stats"], peaks, peak_src, run.label, path_flops, ms_max)
        kernels = kernel_table(prof["stats"], steps)
        launches = head["launches"]
    else:  # graph replays carry no per-launch events: the whole step is the unit
        stats = {"whole step (CUDA graph replay)": {
            "flops": path_flops, "total_ms": ms_max, "launches": run.graph_launches * steps,
            "bytes": 0.0}}
        roof = tensor_roofline(stats, peaks, peak_src, run.label, path_flops, ms_max)
        kernels = {}
        launches = run.graph_launches * steps
    return {"ms": ms_max, "per_step": head["per_step"], "launches": launches,
            "clocks": {**head["clocks"], "remeasured": remeasured}, "roofline": roof,
            "kernels": kernels, "after_headline": between}


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
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    stream = torch.cuda.current_stream(dev)
    timer = Timer(dev, stream, uuid, barrier)
    peaks, peak_src = load_peaks()
    warmup = max(args.warmup, 3)

    run = FlceRun(w, dev, graph=args.graph)
    if args.fused_head_cast:
        if args.graph or w.w_dtype != "f32":
            raise SystemExit("--fused-head-cast needs an FP32-head workload and no --graph")
        run.use_fused_head_cast(dev)
    n = w.n_tokens

    # ---- end to end: pinned host inputs -> device, fwd + bwd, loss -> host, every step.
    # Step k+1's inputs are copied on a second stream into the other of two
    # device buffers while step k computes; every copy is inside the timed
    # region (the copy stream starts after e0, the last step waits for its copy).
    d = run.data
    h_host = d["hidden"].pin_memory()
    l_host = d["labels"].pin_memory()
    loss_host = torch.empty(1, dtype=torch.float32).pin_memory()
    copy_stream = torch.cuda.Stream(dev)
    bufs = [(torch.empty_like(run.hid), torch.empty_like(run.lab)) for _ in range(2)]
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
            run.step(*bufs[b])
            consumed[b].record(stream)
            loss_host.copy_(run.loss, non_blocking=True)

    def after_headline(head):
        # Right after the headline pass, in its power regime: the end-to-end
        # pass, then cuBLAS for as long as the headline took.
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
        return {"e2e_ms": e2e_ms, "cublas": cublas_same_run(dev, stream, head["ms"] / 1e3)}

    m = measure_flce(run, timer, args.steps, warmup, world, max_over_ranks, peaks, peak_src,
                     after_headline=after_headline)
    ref = m["after_headline"]["cublas"]
    m["roofline"]["cublas_same_run"] = ref
    m["roofline"]["frac_of_cublas_same_run"] = m["roofline"]["achieved"] / ref["tflops"]
    value = aggregate_throughput(n, args.steps, world, m["ms"])
    e2e_ms = m["after_headline"]["e2e_ms"]
    e2e_value = aggregate_throughput(n, args.steps, world, e2e_ms)
    h2d = run.hid.numel() * run.hid.element_size() + run.lab.numel() * 8

    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": warmup, "ms_per_step": m["ms"] / args.steps,
            "ms_per_step_median": statistics.median(m["per_step"]),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(w, f"replicas x{world} (one independent batch per GPU)"),
                       **({"cuda_graph": True} if args.graph else {}),
                       **({"head_cast": "fused into the GEMMs"} if run.fused_cast else {})},
            "roofline": m["roofline"],
            "kernels": m["kernels"],
            "kernel_timing": ("per-launch CUDA events in a second pass of the same steps"
                              if not args.graph else "none inside a CUDA graph"),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": 4,
                    "api": "lm_head_projection_flce_b200.flce.forward/backward (C ABI via ctypes)",
                    "overlap": "step k+1's H2D copy on a second stream during step k",
                    "order": "timed right after the headline pass"},
            "gpu_launches": m["launches"],
            "clocks": m["clocks"],
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, d)
    del bufs, h_host, l_host, run
    torch.cuda.empty_cache()

    # ---- the other large workloads and cross entropy on given logits, one GPU only:
    # a short timed pass each, reported under their own key (the headline stays above).
    if world == 1 and not args.no_extras and not args.graph:
        extras = {}
        for wx in (W.SOFTCAP_F32_HEAD, W.LONG_SEQ, W.LARGE_HEAD):
            if wx.name == w.name:
                continue
            rx = FlceRun(wx, dev)
            k = max(5, args.extra_steps)

            def extra_entry(mx, config):
                return {"value": wx.n_tokens * k / (mx["ms"] / 1e3), "unit": UNIT, "steps": k,
                        "warmup": 3, "ms_per_step": mx["ms"] / k,
                        "ms_per_step_median": statistics.median(mx["per_step"]),
                        "config": config, "roofline": mx["roofline"], "kernels": mx["kernels"],
                        "gpu_launches": mx["launches"], "clocks": mx["clocks"]}

            mx = measure_flce(rx, timer, k, 3, 1, lambda x: x, peaks, peak_src)
            entry = extra_entry(mx, workload_config(wx, "one GPU"))
            if not args.no_cpu_baseline:
                entry["cpu_baseline"] = cpu_baseline(wx, rx.data, target_s=6.0)
            extras[wx.name] = entry
            if wx.w_dtype == "f32":
                # the same workload with the head rounded inside the GEMMs (no BF16 copy)
                rx.use_fused_head_cast(dev)
                mx = measure_flce(rx, timer, k, 3, 1, lambda x: x, peaks, peak_src)
                cfg = {**workload_config(wx, "one GPU"), "head_cast": "fused into the GEMMs",
                       "workspace_bytes": int(rx.ws.numel())}
                extras[wx.name + "/fused_head_cast"] = extra_entry(mx, cfg)
            del rx
            torch.cuda.empty_cache()
        extras[W.CE_LOGITS.name] = measure_chunked_ce(
            timer, max(5, args.extra_steps), 3, peaks, peak_src,
            with_cpu_baseline=not args.no_cpu_baseline)
        line["extra_workloads"] = extras

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()
    return 0


def ce_cpu_baseline(d: dict, target_s: float = 6.0) -> dict:
    """The oracle's cross entropy on given logits, timed on a token sample."""
    import numpy as np
    import torch
    from oracle import flce_oracle as O
    z = d["logits"]
    lab = d["labels"].numpy()
    rng = np.random.default_rng(7)
    s = 16
    while True:
        rows = np.sort(rng.choice(z.shape[0], size=s, replace=False))
        zs = z[torch.from_numpy(rows)].double().numpy()
        t0 = time.perf_counter()
        O.ce_forward(zs, lab[rows])
        O.ce_backward(zs, lab[rows])
        dt = time.perf_counter() - t0
        if dt >= target_s / 4 or s >= z.shape[0]:
            break
        s = min(4 * s, z.shape[0])
    return {"value": s / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{s} seeded token rows of the logits through the FP64 oracle's cross "
                       f"entropy forward + backward, {dt:.1f} s (the FP64 upcast of the rows "
                       "excluded)")}


def measure_chunked_ce(timer: "Timer", steps: int, warmup: int, peaks, peak_src,
                       with_cpu_baseline: bool) -> dict:
    """Cross entropy on given logits [4096, 128256] BF16: forward + backward per step."""
    import torch
    from lm_head_projection_flce_b200 import flce
    from lm_head_projection_flce_b200 import workloads as W
    dev = timer.dev
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
    loss = torch.empty(1, device=dev)
    lse = torch.empty(n, device=dev)

    def step():
        flce.ce_forward(z, lab, reduction=w.reduction, num_label_tokens=nlt, workspace=ws,
                        loss=loss, lse=lse)
        flce.ce_backward(z, lab, lse, grad, reduction=w.reduction, num_label_tokens=nlt,
                         dlogits=dz, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    # The steps here are ~0.5 ms, so the per-launch events of the kernel
    # profile would add a few percent: the step time comes from a pass
    # without them, the per-kernel figures from a second, profiled pass.
    head = timer.run(step, steps)
    prof = timer.run(step, steps, profile=True)
    if flce.get_error(dev) != flce.FLCE_OK:
        raise RuntimeError("device error word set during the timed region")
    out = {
        "metric": "cross entropy on given logits, fwd+bwd tokens/sec on 1 B200",
        "value": n * steps / (head["ms"] / 1e3), "unit": UNIT, "steps": steps, "warmup": warmup,
        "ms_per_step": head["ms"] / steps, "ms_per_step_median": statistics.median(head["per_step"]),
        "dtype": "bf16",
        "config": {"workload": w.name, "n_tokens": n, "vocab": v, "logits_dtype": w.dtype,
                   "logits_sigma": w.sigma, "ignore_frac": w.ignore_frac,
                   "reduction": "sum/num_label_tokens",
                   "l2": "inputs larger than L2: 1.05 GB of logits read twice and 1.05 GB of "
                         "gradient written every step"},
        "roofline": hbm_roofline(prof["stats"], peaks, peak_src, w.name, "ce_logits"),
        "kernels": kernel_table(prof["stats"], steps),
        "kernel_timing": "per-launch CUDA events in a second pass of the same steps",
        "gpu_launches": head["launches"],
        "clocks": head["clocks"],
    }
    if with_cpu_baseline:
        out["cpu_baseline"] = ce_cpu_baseline(d)
    del z, dz, ws
    torch.cuda.empty_cache()
    return out


def run_chunked_ce(args) -> int:
    """--path chunked_ce: cross entropy on given logits as the headline line."""
    import torch

    from lm_head_projection_flce_b200 import flce

    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device (sm_100a)")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    from lm_head_projection_flce_b200 import build as B
    B.build()
    flce.load_library()
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    timer = Timer(dev, torch.cuda.current_stream(dev), uuid)
    peaks, peak_src = load_peaks()
    m = measure_chunked_ce(timer, args.steps, max(args.warmup, 3), peaks, peak_src,
                           with_cpu_baseline=not args.no_cpu_baseline)
    line = {"metric": m.pop("metric"), "value": m.pop("value"), "unit": UNIT, "n_gpus": 1,
            **m, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "data": "synthetic"}
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
