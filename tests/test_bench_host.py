"""bench.py host logic on the CPU: the reference arm's JSON line, rank handling,
max-over-ranks timing with two gloo ranks, clock-sample parsing and the
committed-traffic lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

TINY = "tiny_n64_h256_v1024"


def _run(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _run(["--impl", "reference", "--workload", TINY, "--steps", "2", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == TINY


def test_reference_arm_other_ranks_exit_silently():
    r = _run(["--impl", "reference", "--workload", TINY, "--steps", "2", "--warmup", "3"],
             {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.reduce_max(10.0 * (rank + 1) + 0.5, "cpu")
        out.put((rank, mx))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 20.5), (1, 20.5)]


def test_reduce_max_alone_is_identity():
    assert bench.reduce_max(3.25, "cpu") == 3.25


def test_aggregate_throughput_counts_every_rank():
    # 4 ranks x 4096 tokens x 10 steps over the slowest rank's 200 ms
    assert bench.aggregate_throughput(4096, 10, 4, 200.0) == pytest.approx(4096 * 10 * 4 / 0.2)


def test_clock_summary():
    rows = ["0, 1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
            "0, 1800, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "0, 1900, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "garbage"]
    c = bench.ClockSampler.summarize(rows)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]
    bad = bench.ClockSampler.summarize([rows[0].replace("Not Active, Not Active, Not Active, Not Active",
                                                        "Active, Not Active, Not Active, Not Active")])
    assert "hw_slowdown" in bad["reasons"] and bench.BAD_REASONS & set(bad["reasons"])


def test_clock_summary_keeps_the_timed_window():
    row = "0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {cap}, 2026/12/03 07:26:{sec}"
    rows = [row.format(mhz=1965, cap="Not Active", sec="54.100"),      # idle, before the region
            row.format(mhz=1965, cap="Not Active", sec="54.200"),
            row.format(mhz=1290, cap="Active", sec="54.300"),          # under load
            row.format(mhz=1275, cap="Active", sec="54.400")]
    t = bench.ClockSampler.sample_time("2026/12/03 07:26:54.250")
    c = bench.ClockSampler.summarize(rows, (t, t + 0.2))
    assert c["samples"] == 2 and c["sm_mhz"] == 1282.5 and c["reasons"] == ["sw_power_cap"]
    # no sample inside the window: all rows are used rather than none
    assert bench.ClockSampler.summarize(rows, (t + 10, t + 11))["samples"] == 4
    assert bench.ClockSampler.summarize(rows)["samples"] == 4


def test_committed_traffic_needs_matching_sources(tmp_path, monkeypatch):
    f = tmp_path / "t.json"
    dig = bench.kernel_source_digest()
    f.write_text(json.dumps({"records": [
        {"family": "gemm_fwd_lse", "workload": "w1", "source_digest": dig,
         "bytes_per_launch": 123456},
        {"family": "gemm_bwd_dw", "workload": "w1", "source_digest": "0000",
         "bytes_per_launch": 7}]}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(f))
    assert bench.committed_traffic("w1", "gemm_fwd_lse") == 123456.0
    assert bench.committed_traffic("w1", "gemm_bwd_dw") is None     # taken on other sources
    assert bench.committed_traffic("w2", "gemm_fwd_lse") is None
    f.write_text("not json")
    assert bench.committed_traffic("w1", "gemm_fwd_lse") is None


def test_committed_traffic_record_is_well_formed():
    with open(bench.PROFILE_TRAFFIC) as fh:
        recs = json.load(fh)["records"]
    for r in recs:
        assert {"family", "workload", "source_digest", "bytes_per_launch", "command"} <= set(r)
        assert r["bytes_per_launch"] > 0


def _stats(ms_fwd, ms_bwd):
    return {"gemm_fwd_lse": {"launches": 2, "total_ms": ms_fwd, "flops": 2e12, "bytes": 0.0},
            "gemm_bwd_fused": {"launches": 12, "total_ms": ms_bwd, "flops": 12e12, "bytes": 0.0},
            "lse_merge": {"launches": 2, "total_ms": 0.1, "flops": 0.0, "bytes": 1e8}}


def test_tensor_roofline_uses_the_burst_peak_and_refuses_above_one():
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1350.0}
    r = bench.tensor_roofline(_stats(2.0, 10.0), peaks, "measured", "w", 16e12, 12.5)
    assert r["kernel"] == "gemm_bwd_fused" and r["peak"] == 1650.0
    assert r["achieved"] == pytest.approx(12e12 / 10e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1650.0)
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / 1350.0)
    assert r["whole_path_frac"] == pytest.approx(16e12 / 12.5e-3 / 1e12 / 1650.0)
    # a kernel 'faster' than the peak: the fraction is refused, not reported
    fast = bench.tensor_roofline(_stats(0.5, 5.0), peaks, "measured", "w", 16e12, 5.0)
    assert fast["frac"] is None and "frac_refused" in fast


def test_hbm_roofline_refuses_above_one():
    peaks = {"hbm_gbs": 6500.0}
    st = {"ce_logits_fwd": {"launches": 1, "total_ms": 0.2, "flops": 0.0, "bytes": 1e9},
          "ce_logits_bwd": {"launches": 1, "total_ms": 0.4, "flops": 0.0, "bytes": 2e9}}
    r = bench.hbm_roofline(st, peaks, "measured", "w", "ce_logits")
    assert r["kernel"] == "ce_logits_bwd" and r["frac"] == pytest.approx(5000.0 / 6500.0)
    st["ce_logits_fwd"]["total_ms"] = 0.1
    st["ce_logits_bwd"]["total_ms"] = 0.2     # 10000 GB/s: above the copy bandwidth
    assert bench.hbm_roofline(st, peaks, "measured", "w", "ce_logits")["frac"] is None
