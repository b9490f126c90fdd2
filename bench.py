"""Benchmark of one absorbed MLA decode step: mla_absorb_q -> mla_decode_absorb -> mla_out_up.

Workload: DeepSeek-V3 absorbed decode, B=32 sequences per GPU, 4096 cached positions each,
128 heads, d_c=512, d_R=64, bf16 storage / fp32 accumulation (synthetic seeded data).

    python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

One JSON line on rank 0.  `value` = decoded tokens per second over all ranks (each rank runs
its own batch of sequences: batch-sharded replicas, no collective on the data path), timed
on the device with CUDA events around every step, L2 flushed between steps, max over ranks.
`--impl reference` times the CPU oracle on the same workload instead (rank 0 only).
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from head_latent_attention_absorb_b200.configs import V3_DECODE  # noqa: E402
from head_latent_attention_absorb_b200.inputs import make_decode_inputs  # noqa: E402
from head_latent_attention_absorb_b200.shard import max_over_ranks, shard_range  # noqa: E402

METRIC = "MLA absorbed-decode tokens/s and % of roofline (B=32, N=4096, 128 heads)"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one decode launch on this workload,
# from one ncu capture of the decode kernel, valid only for the kernel source it was taken on
# (sha256 prefix of csrc/decode_sm100.cu).
DECODE_TRAFFIC = {"bytes": 155_889_152 + 3_018_496, "source_sha256": "1e2e3f810ae0b3b4"}


def decode_traffic():
    import hashlib
    src = os.path.join(ROOT, "head_latent_attention_absorb_b200", "csrc", "decode_sm100.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return DECODE_TRAFFIC["bytes"] if h == DECODE_TRAFFIC["source_sha256"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def work_per_step(cfg, lengths):
    """Algorithmic FLOPs and bytes of each call of one step (bf16 = 2 bytes)."""
    n_h, d_c, d_r, d_h, d_v, B = cfg.n_h, cfg.d_c, cfg.d_r, cfg.d_h, cfg.d_v, cfg.B
    tot = int(lengths.sum())
    w_half = n_h * d_h * d_c * 2
    return {
        "absorb_q": {"flops": 2 * B * n_h * d_h * d_c, "bytes": w_half + B * n_h * (d_h + d_c) * 2},
        "decode": {"flops": 2 * tot * n_h * (d_c + d_r) + 2 * tot * n_h * d_c,
                   "bytes": tot * (d_c + d_r) * 2 + B * n_h * (d_c + d_r) * 2 + B * n_h * d_c * 2},
        "out_up": {"flops": 2 * B * n_h * d_c * d_v, "bytes": w_half + B * n_h * (d_c + d_v) * 2},
    }


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


def cpu_oracle_rate(x, seconds: float, max_seqs: int):
    """Time the oracle's absorbed decode, one sequence at a time, for about `seconds`."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count()
    cfg = x["cfg"]
    n, t0 = 0, time.perf_counter()
    while n < max_seqs:
        b = n % cfg.B
        L = int(x["lengths"][b])
        O.absorbed_decode(x["q_nope"][b], x["q_pe"][b], x["c_kv"][b, :L], x["k_r"][b, :L], x["w_kv_b"],
                          cfg.scale, cfg.d_v)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return n / dt, n, dt, cores


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: each step = a bounded sample of the workload."""
    if rank != 0:
        return
    cfg = V3_DECODE
    x = make_decode_inputs(cfg)
    # a bounded sample per step: about two minutes for the whole run, at least one sequence
    _, _, t_one, _ = cpu_oracle_rate(x, 1e9, 1)
    per_step = max(1, min(cfg.B, int(args.ref_budget_s / ((args.steps + args.warmup) * t_one))))
    for _ in range(args.warmup):
        cpu_oracle_rate(x, 1e9, per_step)
    times, cores = [], 1
    for _ in range(args.steps):
        rate, n, dt, cores = cpu_oracle_rate(x, 1e9, per_step)
        times.append(dt / n)
    s_per_seq = statistics.mean(times)
    value = 1.0 / s_per_seq
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_per_seq * cfg.B * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "n_max": cfg.n_max, "n_h": cfg.n_h, "d_c": cfg.d_c,
                       "d_r": cfg.d_r, "parallelism": "rank 0 only (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} of the {cfg.B} sequences per step, absorbed fp64 form"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def time_secondary(dev, reps: int, which=("ragged", "sparse", "prefill", "append", "fp8proj", "fp8kv", "sparse_prefill",
                                          "multi")):
    """The other workloads of the hot path, each timed on its own with CUDA events (L2 flushed
    before every launch): the ragged long-context decode, the V3.2 top-k decode, the naive causal
    prefill, the cache append of one new token per sequence in front of the decode, the two
    projections with an FP8 wkv_b, and a V3.2 sparse prefill.  Reported beside the headline line;
    algorithmic bytes / FLOPs as for the headline."""
    from head_latent_attention_absorb_b200 import api
    from head_latent_attention_absorb_b200.configs import PREFILL, RAGGED_LONG, SPARSE_V32
    from head_latent_attention_absorb_b200.inputs import make_prefill_inputs
    peaks = load_peaks()
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps + 3)]
        for e0, e1 in ev:
            flush.zero_()
            e0.record(stream); fn(); e1.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev[3:])

    out = {}
    for cfg in [c for c, k in ((RAGGED_LONG, "ragged"), (SPARSE_V32, "sparse")) if k in which]:
        x = make_decode_inputs(cfg)
        cache = x["cache"].to(dev)
        c_kv, k_r = cache[..., :cfg.d_c], cache[..., cfg.d_c:]
        w = x["w_kv_b"].to(dev)
        qt = api.mla_absorb_q(cfg.dims, x["q_nope"].to(dev), w)
        q_pe, lengths = x["q_pe"].to(dev), x["lengths"].to(dev)
        topk = None if x["topk"] is None else x["topk"].to(dev)
        ctx = torch.empty_like(qt)
        ws = torch.empty((api.mla_decode_workspace_size(cfg.dims, torch.bfloat16, cfg.B, cfg.n_max,
                                                        0 if topk is None else cfg.topk),), dtype=torch.uint8,
                         device=dev)
        ms = timed(lambda: api.mla_decode_absorb(cfg.dims, qt, q_pe, c_kv, k_r, lengths, cfg.scale, topk_idx=topk,
                                                 ctx=ctx, workspace=ws, stream=stream))
        keys = cfg.B * cfg.topk if topk is not None else int(x["lengths"].sum())
        nbytes = keys * (cfg.d_c + cfg.d_r) * 2 + cfg.B * cfg.n_h * (2 * cfg.d_c + cfg.d_r) * 2
        if topk is not None:
            nbytes += cfg.B * cfg.topk * 4
        flops = 2 * keys * cfg.n_h * (2 * cfg.d_c + cfg.d_r)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[cfg.name] = {"call": "mla_decode_absorb", "ms": ms, "tokens_per_s": cfg.B / (ms * 1e-3),
                         "keys": keys, "algorithmic_bytes": nbytes, "achieved_GBs": gbs,
                         "hbm_frac": gbs / peaks["hbm_gbs"], "tflops": flops / (ms * 1e-3) / 1e12}
        del x, cache, c_kv, k_r, ws
        torch.cuda.empty_cache()
    if "append" in which:
        # one new token for each of the decode workload's 32 sequences, written into its cache
        cfg = V3_DECODE
        rng = np.random.default_rng(cfg.seed + 100)
        kv_a = torch.from_numpy(rng.standard_normal((cfg.B, cfg.d_c + cfg.d_r), dtype=np.float32)).to(
            torch.bfloat16).to(dev)
        gain = torch.ones((cfg.d_c,), dtype=torch.float32, device=dev)
        cache = torch.zeros((cfg.B, cfg.n_max, cfg.d_c + cfg.d_r), dtype=torch.bfloat16, device=dev)
        pos = torch.full((cfg.B,), cfg.n_max - 1, dtype=torch.int32, device=dev)
        ms = timed(lambda: api.mla_cache_append(cfg.dims, kv_a, pos, cache[..., :cfg.d_c], cache[..., cfg.d_c:],
                                                gain, stream=stream))
        row = (cfg.d_c + cfg.d_r) * 2
        nbytes = cfg.B * (2 * row + 4) + cfg.d_c * 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        out["append_b32"] = {"call": "mla_cache_append", "ms": ms, "tokens_per_s": cfg.B / (ms * 1e-3),
                             "algorithmic_bytes": nbytes, "achieved_GBs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                             "note": "a few KB per call: bound by launch latency, not by HBM"}
        del cache
        torch.cuda.empty_cache()
    if "multi" in which:
        # two new tokens per sequence (e.g. a speculative token) on the decode workload's cache: each
        # token attends its visible rows; algorithmic bytes count the cache once
        cfg, T = V3_DECODE, 2
        x = make_decode_inputs(cfg)
        cache = x["cache"].to(dev)
        c_kv, k_r = cache[..., :cfg.d_c], cache[..., cfg.d_c:]
        rng = np.random.default_rng(cfg.seed + 400)
        qt = torch.from_numpy(rng.standard_normal((cfg.B, T, cfg.n_h, cfg.d_c), dtype=np.float32) * 0.2).to(
            torch.bfloat16).to(dev)
        qp = torch.from_numpy(rng.standard_normal((cfg.B, T, cfg.n_h, cfg.d_r), dtype=np.float32)).to(
            torch.bfloat16).to(dev)
        lengths = x["lengths"].to(dev)
        ctx = torch.empty((cfg.B, T, cfg.n_h, cfg.d_c), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((api.mla_decode_workspace_size(cfg.dims, torch.bfloat16, cfg.B * T, cfg.n_max),),
                         dtype=torch.uint8, device=dev)
        ms = timed(lambda: api.mla_decode_absorb_multi(cfg.dims, qt, qp, c_kv, k_r, lengths, cfg.scale, ctx=ctx,
                                                       workspace=ws, stream=stream))
        lens = x["lengths"].to(torch.int64)
        keys = int(sum(int(L) - T + 1 + s_ for L in lens for s_ in range(T)))
        nbytes = int(lens.sum()) * (cfg.d_c + cfg.d_r) * 2 + cfg.B * T * cfg.n_h * (2 * cfg.d_c + cfg.d_r) * 2
        flops = 2 * keys * cfg.n_h * (2 * cfg.d_c + cfg.d_r)
        gbs = nbytes / (ms * 1e-3) / 1e9
        tf = flops / (ms * 1e-3) / 1e12
        out["multi_b32_t2_n4096"] = {"call": "mla_decode_absorb_multi", "ms": ms, "tokens_per_s": cfg.B * T / (ms * 1e-3),
                                     "algorithmic_bytes": nbytes, "achieved_GBs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                                     "flops": flops, "tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"],
                                     "roofline_frac": max(nbytes / (peaks["hbm_gbs"] * 1e9),
                                                          flops / (peaks["bf16_tflops"] * 1e12)) / (ms * 1e-3)}
        del x, cache, c_kv, k_r, ws
        torch.cuda.empty_cache()
    if "fp8kv" in which:
        # the decode workload over an FP8 latent cache: packed 656-byte rows (512 E4M3 codes, 4 fp32
        # scales, 64 bf16 rotary features), dequantised on chip
        from head_latent_attention_absorb_b200.inputs import pack_fp8_cache, quantize_latent_fp8
        cfg = V3_DECODE
        x = make_decode_inputs(cfg)
        c8, sc = quantize_latent_fp8(x["c_kv"])
        rows = pack_fp8_cache(c8, sc, x["k_r"]).to(dev)
        c8d, scd, krd = rows[..., :512], rows[..., 512:528].view(torch.float32), rows[..., 528:].view(torch.bfloat16)
        qt = torch.from_numpy(np.random.default_rng(cfg.seed + 500).standard_normal(
            (cfg.B, cfg.n_h, cfg.d_c), dtype=np.float32) * 0.2).to(torch.bfloat16).to(dev)
        qp, lengths = x["q_pe"].to(dev), x["lengths"].to(dev)
        ctx = torch.empty((cfg.B, cfg.n_h, cfg.d_c), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((api.mla_decode_workspace_size(cfg.dims, torch.bfloat16, cfg.B, cfg.n_max),),
                         dtype=torch.uint8, device=dev)
        ms = timed(lambda: api.mla_decode_absorb_fp8kv(cfg.dims, qt, qp, c8d, scd, krd, lengths, cfg.scale, ctx=ctx,
                                                       workspace=ws, stream=stream))
        keys = int(x["lengths"].to(torch.int64).sum())
        nbytes = keys * (cfg.d_c + 16 + cfg.d_r * 2) + cfg.B * cfg.n_h * (cfg.d_c + cfg.d_r + cfg.d_c) * 2
        flops = 2 * keys * cfg.n_h * (2 * cfg.d_c + cfg.d_r)
        gbs = nbytes / (ms * 1e-3) / 1e9
        tf = flops / (ms * 1e-3) / 1e12
        out["fp8kv_b32_n4096"] = {"call": "mla_decode_absorb_fp8kv", "ms": ms, "tokens_per_s": cfg.B / (ms * 1e-3),
                                  "algorithmic_bytes": nbytes, "achieved_GBs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                                  "flops": flops, "tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"],
                                  "roofline_frac": max(nbytes / (peaks["hbm_gbs"] * 1e9),
                                                       flops / (peaks["bf16_tflops"] * 1e12)) / (ms * 1e-3)}
        del x, rows, ws
        torch.cuda.empty_cache()
    if "fp8proj" in which:
        # the two projections of the decode workload with an e4m3 wkv_b and 128 x 128 block scales
        cfg = V3_DECODE
        rng = np.random.default_rng(cfg.seed + 200)
        w = torch.from_numpy(rng.standard_normal((cfg.n_h * (cfg.d_h + cfg.d_v), cfg.d_c), dtype=np.float32) * 0.02)
        amax = w.reshape(w.shape[0] // 128, 128, cfg.d_c // 128, 128).abs().amax(dim=(1, 3)).clamp_min(1e-12)
        scale = (amax / 448.0).float()
        wq = (w / scale.repeat_interleave(128, 0).repeat_interleave(128, 1)).to(torch.float8_e4m3fn).to(dev)
        scale = scale.to(dev)
        q_nope = torch.from_numpy(rng.standard_normal((cfg.B, cfg.n_h, cfg.d_h), dtype=np.float32)).to(
            torch.bfloat16).to(dev)
        ctx = torch.from_numpy(rng.standard_normal((cfg.B, cfg.n_h, cfg.d_c), dtype=np.float32) * 0.05).to(
            torch.bfloat16).to(dev)
        qt = torch.empty((cfg.B, cfg.n_h, cfg.d_c), dtype=torch.bfloat16, device=dev)
        o = torch.empty((cfg.B, cfg.n_h, cfg.d_v), dtype=torch.bfloat16, device=dev)
        half_w = cfg.n_h * cfg.d_h * cfg.d_c  # fp8 bytes of one projection's weight half
        for name, fn, nbytes in (
                ("absorb_q_fp8", lambda: api.mla_absorb_q_fp8(cfg.dims, q_nope, wq, scale, q_tilde=qt, stream=stream),
                 half_w + cfg.B * cfg.n_h * (cfg.d_h + cfg.d_c) * 2),
                ("out_up_fp8", lambda: api.mla_out_up_fp8(cfg.dims, ctx, wq, scale, out=o, stream=stream),
                 half_w + cfg.B * cfg.n_h * (cfg.d_c + cfg.d_v) * 2)):
            ms = timed(fn)
            gbs = nbytes / (ms * 1e-3) / 1e9
            out[name + "_b32"] = {"call": "mla_" + name, "ms": ms, "algorithmic_bytes": nbytes, "achieved_GBs": gbs,
                                  "hbm_frac": gbs / peaks["hbm_gbs"]}
        del wq
        torch.cuda.empty_cache()
    if "sparse_prefill" in which:
        # a V3.2-style sparse prefill: B=1, S=8192, each row's 2048 selected positions (itself plus
        # 2047 drawn over the sequence; the causal mask removes the later ones)
        cfg = PREFILL.with_(B=1, n_max=8192)
        p = make_prefill_inputs(cfg)
        S, k = cfg.n_max, 2048
        rng = np.random.default_rng(cfg.seed + 300)
        topk = np.empty((1, S, k), dtype=np.int32)
        for s_ in range(S):
            topk[0, s_, 0] = s_
            topk[0, s_, 1:] = rng.choice(S, k - 1, replace=False)
        visible = sum(len({t for t in topk[0, s_].tolist() if t <= s_}) for s_ in range(S))
        q, c_kv, k_r, w = p["q"].to(dev), p["c_kv"].to(dev), p["k_r"].to(dev), p["w_kv_b"].to(dev)
        tk = torch.from_numpy(topk).to(dev)
        o = torch.empty((1, S, cfg.n_h, cfg.d_v), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((int(api.lib().mla_prefill_sparse_workspace_size(api._dims(cfg.dims), 1, 1, S)),),
                         dtype=torch.uint8, device=dev)
        ms = timed(lambda: api.mla_prefill_sparse(cfg.dims, q, c_kv, k_r, w, cfg.scale, tk, out=o, workspace=ws,
                                                  stream=stream))
        flops = 2 * S * cfg.n_h * (cfg.d_h + cfg.d_v) * cfg.d_c + 2 * cfg.n_h * visible * ((cfg.d_h + cfg.d_r) + cfg.d_v)
        tf = flops / (ms * 1e-3) / 1e12
        out["sparse_prefill_b1_s8192_k2048"] = {"call": "mla_prefill_sparse", "ms": ms, "visible_pairs": visible,
                                                "flops": flops, "tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"]}
        del q, c_kv, k_r, w, tk, o, ws
        torch.cuda.empty_cache()
    if "prefill" not in which:
        return out
    cfg = PREFILL
    p = make_prefill_inputs(cfg)
    q, c_kv, k_r, w = p["q"].to(dev), p["c_kv"].to(dev), p["k_r"].to(dev), p["w_kv_b"].to(dev)
    o = torch.empty((cfg.B, cfg.n_max, cfg.n_h, cfg.d_v), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((api.mla_prefill_workspace_size(cfg.dims, torch.bfloat16, cfg.B, cfg.n_max),),
                     dtype=torch.uint8, device=dev)
    ms = timed(lambda: api.mla_prefill_naive(cfg.dims, q, c_kv, k_r, w, cfg.scale, out=o, workspace=ws,
                                             stream=stream))
    S, B = cfg.n_max, cfg.B
    flops = 2 * B * S * cfg.n_h * (cfg.d_h + cfg.d_v) * cfg.d_c \
        + 2 * B * cfg.n_h * (S * (S + 1) // 2) * ((cfg.d_h + cfg.d_r) + cfg.d_v)
    tf = flops / (ms * 1e-3) / 1e12
    out[cfg.name] = {"call": "mla_prefill_naive", "ms": ms, "tokens_per_s": B * S / (ms * 1e-3), "flops": flops,
                     "tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"]}
    return out


def run_ours(args, rank, world, local_rank):
    from head_latent_attention_absorb_b200 import api
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = V3_DECODE
    # this rank's share of the global batch (world x B sequences); each share has its own cache
    first_seq, n_seq = shard_range(world * cfg.B, world, rank)
    assert n_seq == cfg.B
    x = make_decode_inputs(cfg, seed=cfg.seed + first_seq)
    dims = cfg.dims
    B = cfg.B
    cache = x["cache"].to(dev)
    c_kv, k_r = cache[..., :cfg.d_c], cache[..., cfg.d_c:]
    w = x["w_kv_b"].to(dev)
    q_nope, q_pe, lengths = x["q_nope"].to(dev), x["q_pe"].to(dev), x["lengths"].to(dev)
    q_tilde = torch.empty((B, cfg.n_h, cfg.d_c), dtype=torch.bfloat16, device=dev)
    ctx = torch.empty_like(q_tilde)
    lse = torch.empty((B, cfg.n_h), dtype=torch.float32, device=dev)
    out = torch.empty((B, cfg.n_h, cfg.d_v), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((api.mla_decode_workspace_size(dims, torch.bfloat16, B, cfg.n_max),), dtype=torch.uint8,
                     device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty((L2_FLUSH_BYTES,), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    n_launch = 2 + api.mla_decode_num_launches(dims, torch.bfloat16, B, cfg.n_max)

    def step_on(st, qn, qp, marks=False):
        api.mla_absorb_q(dims, qn, w, q_tilde, stream=st)
        if marks:
            ev[1].record(st)
        api.mla_decode_absorb(dims, q_tilde, qp, c_kv, k_r, lengths, cfg.scale, ctx=ctx, lse=lse, workspace=ws,
                              dev_err=err, stream=st)
        if marks:
            ev[2].record(st)
        api.mla_out_up(dims, ctx, w, out, stream=st)

    def step(qn, qp):
        step_on(stream, qn, qp, marks=True)

    # ---- per-call timing (each call launched on its own, events between the calls) ------------
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K + args.warmup)]
    for i in range(args.warmup + K):
        ev = evs[i]
        flush.zero_()
        ev[0].record(stream); step(q_nope, q_pe); ev[3].record(stream)
    torch.cuda.synchronize()
    per = {"absorb_q": [], "decode": [], "out_up": []}
    for ev in evs[args.warmup:]:
        per["absorb_q"].append(ev[0].elapsed_time(ev[1]))
        per["decode"].append(ev[1].elapsed_time(ev[2]))
        per["out_up"].append(ev[2].elapsed_time(ev[3]))
    ms = {k: statistics.mean(v) for k, v in per.items()}

    # ---- the step as a server runs it: the three calls captured once in a CUDA graph and
    # replayed (no host work between the kernels); CUDA events around every replay --------------
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(graph, stream=cap):
            step_on(cap, q_nope, q_pe)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K + args.warmup)]
    for i in range(args.warmup):
        flush.zero_()
        gev[i][0].record(stream); graph.replay(); gev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_wall = time.perf_counter()
        for i in range(args.warmup, args.warmup + K):
            flush.zero_()
            gev[i][0].record(stream); graph.replay(); gev[i][1].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms["step"] = statistics.mean(e[0].elapsed_time(e[1]) for e in gev[args.warmup:])
    assert api.mla_get_device_error(err) == 0, "device error flag raised during the bench"

    # ---- end to end through the public API with host buffers ---------------------------------
    qn_h = x["q_nope"].pin_memory()
    qp_h = x["q_pe"].pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    qn_d, qp_d = torch.empty_like(q_nope), torch.empty_like(q_pe)
    h2d = qn_h.numel() * qn_h.element_size() + qp_h.numel() * qp_h.element_size()
    d2h = out_h.numel() * out_h.element_size()
    e2e_ms = []
    for i in range(args.warmup + K):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        qn_d.copy_(qn_h, non_blocking=True)
        qp_d.copy_(qp_h, non_blocking=True)
        step(qn_d, qp_d)
        out_h.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e = statistics.mean(e2e_ms)

    # ---- max over ranks -----------------------------------------------------------------------
    ms_step, ms_dec, ms_e2e, ms_abs, ms_up = max_over_ranks(
        [ms["step"], ms["decode"], e2e, ms["absorb_q"], ms["out_up"]], device=dev)
    if rank != 0:
        return

    peaks = load_peaks()
    work = work_per_step(cfg, x["lengths"])
    dec = work["decode"]
    achieved_gbs = dec["bytes"] / (ms_dec * 1e-3) / 1e9
    achieved_tf = dec["flops"] / (ms_dec * 1e-3) / 1e12
    clocks = clk.summary()
    cpu_rate, cpu_n, cpu_dt, cores = cpu_oracle_rate(x, args.cpu_seconds, 10 ** 6)
    line = {
        "metric": METRIC, "value": world * B / (ms_step * 1e-3), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "B_per_gpu": B, "n_max": cfg.n_max, "n_h": cfg.n_h, "d_c": cfg.d_c,
                   "d_r": cfg.d_r, "d_h": cfg.d_h, "d_v": cfg.d_v, "global_batch": world * B,
                   "parallelism": f"batch-sharded replicas x{world}", "l2": "flushed (256 MiB write) before each step",
                   "timing": "CUDA events around each replay of the step's CUDA graph (the three calls "
                             "captured once), mean over steps, max over ranks; per-call times from separate "
                             "launches with events between the calls"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": decode_traffic(), "kernel": "mla_decode_absorb",
                     "peak_source": peaks["source"] + " (hbm_gbs, burst)",
                     "algorithmic_bytes_per_launch": dec["bytes"], "ms_per_launch": ms_dec,
                     "tensor_achieved_tflops": achieved_tf, "tensor_peak_tflops": peaks["bf16_tflops"],
                     "tensor_frac": achieved_tf / peaks["bf16_tflops"]},
        "per_call_ms": {"absorb_q": ms_abs, "decode": ms_dec, "out_up": ms_up},
        "cpu_baseline": {"value": cpu_rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{cpu_n} sequences of this workload, fp64 absorbed form, {cpu_dt:.1f} s"},
        "e2e": {"value": world * B / (ms_e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": "queries copied from pinned host memory and outputs read back every step; cache and "
                        "wkv_b resident"},
        "gpu_launches": n_launch * K,
        "secondary": None if args.no_secondary else time_secondary(dev, 10),
        "clocks": clocks,
        "wall_s_timed_region": t_wall,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-budget-s", type=float, default=120.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the timings of the secondary workloads (ragged, top-k, prefill, cache append, "
                         "FP8 projections, sparse prefill)")
    ap.add_argument("--only", choices=["ragged", "sparse", "prefill", "append", "fp8proj", "fp8kv", "sparse_prefill", "multi"],
                    help="time only this secondary workload (--steps launches after 3 warm-up ones) and print "
                         "its entry; a small command for profilers, not a bench line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.only:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(time_secondary(dev, args.steps, (args.only,))))
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
