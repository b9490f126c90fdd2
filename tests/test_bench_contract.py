"""bench.py's reference arm (the CPU oracle timed on the host cores) prints one JSON line with the
keys the benchmark contract names; it runs without a GPU."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-budget-s", "2"], capture_output=True, text=True, cwd=ROOT,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] >= 3
    assert d["value"] > 0 and d["unit"] == d["e2e"]["unit"] and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"] == "v3_decode_b32_n4096"


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_algorithmic_work_of_the_step():
    """The roofline numerators for the benchmarked step (B = 32, N = 4096, DeepSeek-V3 dimensions):
    the decode reads the 576-feature cache rows once (150,994,944 B), the query rows (q~ and q^R) and
    writes ctx; the two projections each read one 16.8 MB half of wkv_b."""
    import torch
    bench = _bench_module()
    cfg = bench.V3_DECODE
    w = bench.work_per_step(cfg, torch.full((32,), 4096, dtype=torch.int32))
    assert w["decode"]["bytes"] == 32 * 4096 * 576 * 2 + 32 * 128 * 576 * 2 + 32 * 128 * 512 * 2 == 159_907_840
    assert w["decode"]["flops"] == 2 * 131072 * 128 * (576 + 512) == 36_507_222_016
    for call in ("absorb_q", "out_up"):
        assert w[call]["bytes"] == 128 * 128 * 512 * 2 + 32 * 128 * (128 + 512) * 2 == 22_020_096
        assert w[call]["flops"] == 2 * 32 * 128 * 128 * 512
    # ragged lengths count only the cached rows
    w2 = bench.work_per_step(cfg.with_(B=2), torch.tensor([1, 100], dtype=torch.int32))
    assert w2["decode"]["bytes"] == 101 * 576 * 2 + 2 * 128 * 576 * 2 + 2 * 128 * 512 * 2


def test_decode_traffic_tied_to_the_kernel_source(monkeypatch):
    """The ncu traffic figure is reported only for the decode source it was captured on, and then it
    is close to the algorithmic bytes (no re-reads)."""
    bench = _bench_module()
    t = bench.decode_traffic()
    assert t is None or abs(t / 159_907_840 - 1) < 0.05
    monkeypatch.setitem(bench.DECODE_TRAFFIC, "source_sha256", "0" * 16)
    assert bench.decode_traffic() is None


def test_clock_summary_parsing():
    """nvidia-smi samples taken during the timed region: median SM clock, throttle reasons that were
    active in any sample, and an explicit 'unsampled' when nothing was read."""
    bench = _bench_module()
    c = bench.ClockSampler(0)
    c.out = ("0, 1965, 1965, 400.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
             "0, 1800, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 1900, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    s = c.summary()
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 980.0
    c.out = ""
    assert c.summary()["reasons"] == ["unsampled"]
