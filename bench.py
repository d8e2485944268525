#!/usr/bin/env python
"""Latent-KV decode throughput of libtpla on B200.

One step = one pass of the whole decode hot path over one batch of the
DeepSeek-V3-shaped workload (B=64 requests, H=128 heads, 32768 cached
tokens each, paged 64-token blocks, 576 bf16 values per token):
  tpla_decode_ex (TPLA, G shards, split-KV + log-sum-exp merge inside)
  -> tpla_vup_combine (V up-projection; stands in for the TP all-reduce).
The Walsh-Hadamard reparameterisation is applied once to q, the cache and
(folded) W_uv before timing, as a deployment folds it into the weights.

Metric: latent-KV GB/s = algorithmic cache bytes per step / step time
(also decode tokens/s per layer).  Inputs (2.4 GB) exceed the 126 MB L2, so
no flush is needed between steps.  Multi-GPU runs are independent replicas
(the decode path has no cross-GPU exchange).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_latent_kv_dim_b200.replicas import aggregate_rate, max_over_ranks  # noqa: E402
from mla_latent_kv_dim_b200.workloads import (LATENT, ROPE, WIDTH, CONFIGS,  # noqa: E402
                                              make_workload)

METRIC = "latent-KV GB/s & decode tok/s/layer at H=128 L=32K (% HBM peak), vs G"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (DGX figure); context beside the measured copy


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="dsv3", choices=sorted(CONFIGS))
    ap.add_argument("--G", type=int, default=2)
    ap.add_argument("--rope", default="replicate", choices=["replicate", "split"])
    ap.add_argument("--no-hadamard", action="store_true")
    ap.add_argument("--kernel", default="auto", choices=["auto", "generic", "sm100"])
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the per-G sweep and the other workloads")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (V2-Lite, Kimi-K2, long context)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--batch", type=int, default=None,
                    help="fewer requests of the same shape (profiling captures)")
    ap.add_argument("--prefill", type=int, default=0,
                    help="with --profile: time tpla_prefill of one prompt of this many "
                         "tokens (H = 128) instead of the decode")
    ap.add_argument("--profile", action="store_true",
                    help="decode launches only: warmup + steps, one short JSON line")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_per_token_head(G, shard=None, rope_mode="replicate"):
    """Algorithmic MMA flops per (token, head): QK over each shard's key
    columns plus PV over its latent columns."""
    d = LATENT // G
    r = ROPE if rope_mode == "replicate" else ROPE // G
    shards = G if shard is None else 1
    return shards * (2 * (d + r) + 2 * d)


def one_shard_speedups(vs_G):
    """Decode time of exact MLA (G=1, every latent column) over the time of
    one TPLA shard's read (one-shard mode), per G: the per-rank attention
    speedup that the pages' end-to-end TPLA-vs-MLA decode speedups at 32K
    context stem from.  None without a G=1 entry."""
    t = {(e["G"], e["mode"]): e["decode_us"] for e in vs_G}
    base = t.get((1, "full"))
    if not base:
        return None
    return {f"G{g}": round(base / t[(g, "one-shard")], 3)
            for g in sorted({e["G"] for e in vs_G}) if (g, "one-shard") in t}


def decode_kernel_hash():
    h = hashlib.sha256()
    for f in ("decode_sm100.cu", "decode_generic.cu", "merge.cu"):
        p = os.path.join(ROOT, "mla_latent_kv_dim_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_name, workload):
    """Per-launch DRAM bytes of the decode kernel from a committed ncu summary,
    if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(kernel_name, {}).get(workload)
        if e and e.get("source_hash") == decode_kernel_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region: NVML
    every 2 ms when available (a timed region is tens of milliseconds), else
    nvidia-smi at its 100 ms minimum."""

    # NVML clocks-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.nvml = None
        self.samples = []
        self.lines = []
        self.stop_flag = False

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.hdl = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.hdl, pynvml.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _poll(self):
        n = self.nvml
        while not self.stop_flag:
            try:
                self.samples.append((n.nvmlDeviceGetClockInfo(self.hdl, n.NVML_CLOCK_SM),
                                     n.nvmlDeviceGetCurrentClocksEventReasons(self.hdl)))
            except Exception:
                break
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.stop_flag = True
            self.t.join(timeout=2)
            sm = [float(c) for c, _ in self.samples]
            reasons = set()
            for _, r in self.samples:
                for bit, name in self.REASONS.items():
                    if r & bit:
                        reasons.add(name)
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_max_mhz": float(self.max_mhz), "reasons": sorted(reasons),
                    "samples": len(sm), "source": "nvml 2 ms"}
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi 100 ms"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, G, rope, hadamard, budget_s, prepared=None):
    """Time the float64 oracle on whole requests of the workload, doing what
    one GPU step does per request: decode (on the stored, already rotated
    cache when the Hadamard is folded in) and the V-up combine.  The rotation
    itself is set-up on both sides and is not timed.  Runs until about
    ``budget_s`` seconds of oracle time have passed.  ``prepared`` (a dict)
    keeps each request's gathered, rotated rows between calls, as the stored
    cache stays between GPU steps.  Returns (GB/s, seconds, requests)."""
    from oracle import tpla_oracle as O  # CPU baseline leg only
    from mla_latent_kv_dim_b200.workloads import as_f64
    Wv = as_f64(w.W_uv) if w.W_uv is not None else None
    if Wv is not None and hadamard:  # folded V-up weights, as the GPU step uses
        Wv = np.swapaxes(O.hadamard_ref(np.swapaxes(Wv, 1, 2), 512), 1, 2)
    done_bytes = 0
    t_total = 0.0
    reqs = 0
    b = 0
    while t_total < budget_s and b < w.B:
        L = int(w.seq_lens[b])
        if prepared is not None and b in prepared:
            q, rows = prepared[b]
        else:
            pages = (L + 63) // 64
            if w.page_table is not None:
                rows = as_f64(w.cache[w.page_table[b, :pages].long()].reshape(pages * 64,
                                                                              WIDTH)[:L])
            else:
                rows = as_f64(w.cache[b, :L])
            q = as_f64(w.q[b:b + 1])
            if hadamard:
                q = O.hadamard_ref(q, 512)
                rows = O.hadamard_ref(rows, 512)
            if prepared is not None:
                prepared[b] = (q, rows)
        t0 = time.perf_counter()
        out, _ = O.tpla_decode_ref(q, [rows], G, rope, np.float32(w.scale))
        if Wv is not None:
            O.vup_ref(out, Wv)
        t_total += time.perf_counter() - t0
        done_bytes += L * WIDTH * 2
        reqs += 1
        b += 1
    return done_bytes / t_total / 1e9, t_total, reqs


# ------------------------------------------------------------------ reference arm

def step_config(args, w, kernel, parallelism):
    """The workload description both arms print."""
    cache_bytes = w.latent_kv_bytes(1)
    l2 = (f"inputs {cache_bytes / 1e9:.1f} GB > 126 MB L2; no flush needed"
          if cache_bytes > 126e6 else
          f"inputs {cache_bytes / 1e6:.0f} MB fit in the 126 MB L2 (not flushed)")
    return {"workload": args.config, "B": w.B, "H": w.H, "seq_len": int(w.seq_lens.max()),
            "G": args.G, "rope_mode": args.rope, "hadamard": not args.no_hadamard,
            "paged_block": 64 if w.page_table is not None else None, "kernel": kernel,
            "num_splits": args.num_splits or "auto",
            "step": "decode (+LSE merge) + V-up combine", "l2": l2,
            "parallelism": parallelism}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_workload(args.config)
    hadamard = not args.no_hadamard
    per_step = []
    reqs = 0
    prepared = {}
    for i in range(args.warmup + args.steps):
        gbs, t, n = oracle_sample(w, args.G, args.rope, hadamard,
                                  budget_s=max(0.5, 120.0 / (args.warmup + args.steps)),
                                  prepared=prepared)
        if i >= args.warmup:
            per_step.append(gbs)
            reqs = n
    v = statistics.mean(per_step)
    cores = blas_threads()
    sample = (f"{reqs} request(s) x {w.H} heads x {int(w.seq_lens[0])} tokens of the "
              f"{args.config} workload per step, G={args.G}, decode + V-up on the stored "
              f"cache (set-up rotation not timed), float64 NumPy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(w.latent_kv_bytes(args.G) / (v * 1e9) * 1e3, 1),
        "ms_per_step_note": "one full step extrapolated from the sampled requests",
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no checkpoints or datasets)",
        "config": step_config(args, w, "float64 NumPy oracle (CPU)", "rank 0 only"),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import mla_latent_kv_dim_b200 as tp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    hadamard = not args.no_hadamard
    G, rope = args.G, args.rope

    w = make_workload(args.config, pin=True)
    q = w.q.to(dev)
    cache = w.cache.to(dev, non_blocking=True)
    seq = w.seq_lens.to(dev)
    pt = None if w.page_table is None else w.page_table.to(dev)
    W = w.W_uv.to(dev) if w.W_uv is not None else None
    if W is None:
        g = torch.Generator().manual_seed(1234)
        W = (0.02 * torch.randn((w.H, LATENT, 128), generator=g)).to(torch.bfloat16).to(dev)
    if hadamard:
        # one-off reparameterisation: q, cache and the folded V up-projection
        tp.hadamard_apply(q, LATENT)
        tp.hadamard_apply(cache, LATENT)
        Wt = W.transpose(1, 2).contiguous()
        tp.hadamard_apply(Wt, LATENT)
        W = Wt.transpose(1, 2).contiguous()
    torch.cuda.synchronize()
    B, H = w.B, w.H
    out = torch.empty((B, H, LATENT), dtype=torch.float32, device=dev)
    lse = torch.empty((B, H, G), dtype=torch.float32, device=dev)
    y = torch.empty((B, H, W.shape[2]), dtype=torch.float32, device=dev)
    need = tp.decode_workspace_size(q, cache, seq, pt, G, rope, out, num_splits=args.num_splits,
                                    kernel=args.kernel)
    ws = torch.empty(max(16, need), dtype=torch.uint8, device=dev)
    bytes_step = w.latent_kv_bytes(G)
    flops_step = float(w.seq_lens.to(torch.int64).sum()) * H * flops_per_token_head(G, None, rope)
    stream = torch.cuda.current_stream()

    def decode_once(qq, o, l, shard=None, GG=G):
        tp.decode(qq, cache, seq, pt, GG, rope, w.scale, out=o, lse=l, shard=shard,
                  num_splits=args.num_splits, kernel=args.kernel, workspace=ws)

    def step(ev_a=None, ev_b=None):
        if ev_a is not None:
            ev_a.record(stream)
        decode_once(q, out, lse)
        if ev_b is not None:
            ev_b.record(stream)
        tp.vup_combine(out, W, y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    n0 = tp.launch_count()
    t_start.record(stream)
    for i in range(args.steps):
        step(*evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    n_launch = tp.launch_count() - n0
    clk = clocks.stop()
    if dist:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms, dec_ms = max_over_ranks([ms, dec_ms], dist, dev)
    rate, t_step = aggregate_rate(world, bytes_step, ms, args.steps)
    value = rate / 1e9
    tok_s = world * B / t_step

    # ---- end to end through the public API: host q in, host y out.  Steps
    # are pipelined the way a serving loop would run them: step i's inputs
    # are copied in (one stream) while step i-1 computes (the compute
    # stream) and step i-2's output is copied out (a third stream); two sets
    # of device buffers, events order the reuse.
    q_host = q.cpu().pin_memory()
    seq_host = w.seq_lens.pin_memory()
    pt_host = None if w.page_table is None else w.page_table.pin_memory()
    nbuf = 2
    q_in = [torch.empty_like(q) for _ in range(nbuf)]
    seq_in = [torch.empty_like(seq) for _ in range(nbuf)]
    pt_in = [None if pt is None else torch.empty_like(pt) for _ in range(nbuf)]
    y_dev = [torch.empty_like(y) for _ in range(nbuf)]
    y_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(nbuf)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_comp = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def e2e_step(i):
        k = i % nbuf
        with torch.cuda.stream(s_in):
            if i >= nbuf:
                s_in.wait_event(ev_comp[k])  # step i - 2 no longer reads these inputs
            q_in[k].copy_(q_host, non_blocking=True)
            seq_in[k].copy_(seq_host, non_blocking=True)
            if pt_host is not None:
                pt_in[k].copy_(pt_host, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= nbuf:
            stream.wait_event(ev_out[k])  # step i - 2's output has left the device
        tp.decode(q_in[k], cache, seq_in[k], pt_in[k], G, rope, w.scale, out=out, lse=lse,
                  num_splits=args.num_splits, kernel=args.kernel, workspace=ws)
        tp.vup_combine(out, W, y_dev[k])
        ev_comp[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            y_host[k].copy_(y_dev[k], non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    # the same steps with every copy serialised against the compute (one stream)
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(args.steps):
        q_in[0].copy_(q_host, non_blocking=True)
        seq_in[0].copy_(seq_host, non_blocking=True)
        if pt_host is not None:
            pt_in[0].copy_(pt_host, non_blocking=True)
        tp.decode(q_in[0], cache, seq_in[0], pt_in[0], G, rope, w.scale, out=out, lse=lse,
                  num_splits=args.num_splits, kernel=args.kernel, workspace=ws)
        tp.vup_combine(out, W, y_dev[0])
        y_host[0].copy_(y_dev[0], non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    es_ms = e2.elapsed_time(e3)
    e_ms, es_ms = max_over_ranks([e_ms, es_ms], dist, dev)
    e2e_val = aggregate_rate(world, bytes_step, e_ms, args.steps)[0] / 1e9
    e2e_serial = aggregate_rate(world, bytes_step, es_ms, args.steps)[0] / 1e9
    h2d = q.numel() * 2 + seq.numel() * 4 + (pt.numel() * 4 if pt is not None else 0)
    d2h = y.numel() * 4

    # ---- roofline of the dominant kernel (decode), live CUDA-event timing
    dec_s = dec_ms / 1e3
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # the timed region is tens of milliseconds at full clock: the burst GEMM peak applies
    tc_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved_gbs = bytes_step / dec_s / 1e9
    achieved_tf = flops_step / dec_s / 1e12
    t_hbm = bytes_step / (hbm_peak * 1e9)
    t_tc = flops_step / (tc_peak * 1e12)
    used = "sm100" if args.kernel != "generic" and _sm100_used(tp, q, cache, seq, pt, G, rope, out,
                                                                args) else "generic"
    # G >= 2 runs the shard kernel (one CTA per TPLA shard), G = 1 the pair kernel
    kname = (("tpla_decode_shard" if G >= 2 else "tpla_decode_sm100") if used == "sm100"
             else "decode_generic_kernel")
    traffic = recorded_traffic(kname, args.config)
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": round(achieved_tf, 2), "peak": tc_peak,
                "unit": "TFLOP/s", "frac": round(achieved_tf / tc_peak, 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved_gbs / hbm_peak, 4)}
    roof.update({"traffic": traffic, "kernel": kname,
                 "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
                 "hbm_gbs": round(achieved_gbs, 1), "hbm_frac": round(achieved_gbs / hbm_peak, 4),
                 "hbm_frac_nominal_8tbs": round(achieved_gbs / NOMINAL_HBM_GBS, 4),
                 "tensor_tflops": round(achieved_tf, 2),
                 "tensor_frac_burst": round(achieved_tf / tc_peak, 4),
                 "bytes_per_launch": bytes_step, "flops_per_launch": flops_step,
                 "decode_ms": round(dec_ms, 4)})

    # ---- per-G decode-only sweep (vs G), full and one-shard
    vs_G = []
    tp_rank = None
    setup = None
    clk_extras = None
    if not args.no_extras:
        cs = ClockSampler(local)
        cs.start()
        time.sleep(0.2)
        for GG, shard in ((1, None), (2, None), (4, None), (2, 0), (4, 0)):
            width = LATENT if shard is None else LATENT // GG
            o2 = torch.empty((B, H, width), dtype=torch.float32, device=dev)
            l2 = torch.empty((B, H, GG if shard is None else 1), dtype=torch.float32, device=dev)
            for _ in range(3):
                decode_once(q, o2, l2, shard, GG)
            a = torch.cuda.Event(enable_timing=True)
            bb = torch.cuda.Event(enable_timing=True)
            n = 50
            a.record(stream)
            for _ in range(n):
                decode_once(q, o2, l2, shard, GG)
            bb.record(stream)
            torch.cuda.synchronize()
            t = a.elapsed_time(bb) / 1e3 / n
            nb = w.latent_kv_bytes(GG, shard, rope)
            vs_G.append({"G": GG, "mode": "full" if shard is None else "one-shard",
                         "bytes": nb, "decode_us": round(t * 1e6, 1),
                         "GB_s": round(nb / t / 1e9, 1),
                         "hbm_frac": round(nb / t / 1e9 / hbm_peak, 4),
                         "tok_s_layer": round(B / t, 1)})
            del o2, l2
        # one tensor-parallel rank's step (its one-shard decode + its partial V
        # up-projection, K = 512/G), against the exact-MLA step on one GPU
        # (G = 1 decode + V-up); the all-reduce of y between ranks is not timed
        from mla_latent_kv_dim_b200 import tensor_parallel as TPar
        tp_rank = []
        for GG in (1, 2, 4):
            def rank_step():
                TPar.rank_partial(q, cache, seq, pt, GG, 0, W, w.scale, rope, workspace=ws)
            for _ in range(3):
                rank_step()
            a = torch.cuda.Event(enable_timing=True)
            bb = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(50):
                rank_step()
            bb.record(stream)
            torch.cuda.synchronize()
            tp_rank.append({"G": GG, "rank_step_us": round(a.elapsed_time(bb) / 50 * 1e3, 1),
                            "bytes": w.latent_kv_bytes(GG, 0 if GG > 1 else None, rope)})
        clk_extras = cs.stop()
        setup = setup_ops(tp, dev, cache, w.cache, hbm_peak)

    configs = None
    if not args.no_extras and not args.no_configs and world == 1:
        del cache, q, ws, out, y
        torch.cuda.empty_cache()
        configs = other_workloads(tp, dev, hbm_peak, tc_peak)
        configs["prefill"] = prefill_workload(tp, dev, tc_peak)

    cpu = None
    if rank == 0 and world == 1:
        torch.cuda.synchronize()
        gbs, secs, reqs = oracle_sample(w, G, rope, hadamard, args.cpu_seconds)
        cpu = {"value": round(gbs, 5), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{reqs} whole request(s) x {H} heads x {int(w.seq_lens[0])} tokens, "
                         f"G={G}, {'Hadamard-rotated cache (rotation not timed), ' if hadamard else ''}"
                         f"decode + V-up, {secs:.1f} s of float64 NumPy"}

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; no checkpoints or datasets)",
        "config": step_config(args, w, used, f"replicas x{world}"),
        "tok_s_layer": round(tok_s, 1),
        "hbm_frac_step": round(value / world / hbm_peak, 4),
        "roofline": roof, "vs_G": vs_G, "vs_G_clocks": clk_extras,
        "one_shard_speedup_vs_mla": one_shard_speedups(vs_G),
        "tp_rank_step": tp_rank,
        "setup_ops": setup,
        "configs": configs,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "pipelining": "H2D, compute and D2H on three streams, two buffer sets",
                "serial_value": round(e2e_serial, 2),
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / args.steps, 4)},
        "gpu_launches": n_launch, "clocks": clk,
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 * 2 ** 20


def other_workloads(tp, dev, hbm_peak, tc_peak):
    """Decode (and V-up) timings of the other configured workloads, each on
    its own seeded inputs with the Hadamard reparameterisation folded in:
    DeepSeek-V2-Lite shape (G=2), Kimi-K2 shape (G=1/2/4, both rope modes,
    V-up combine), long context (B=4, 131072 tokens; automatic split against
    32/64/128 explicit chunks, G=1/4).  A cache smaller than twice the L2 is
    timed launch by launch with the L2 flushed in between (a 256 MB write
    outside the timed events); the others stream more than L2 holds."""
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    plan = {
        "v2lite": [dict(G=2, rope="replicate", splits=0, vup=True)],
        "kimi": [dict(G=G, rope=r, splits=0, vup=True) for G in (1, 2, 4)
                 for r in ("replicate", "split")],
        "long": [dict(G=G, rope="replicate", splits=sp, vup=False) for G in (1, 4)
                 for sp in (0, 32, 64, 128)],
    }
    res = {}
    for name, settings in plan.items():
        w = make_workload(name)
        q = w.q.to(dev)
        cache = w.cache.to(dev)
        seq = w.seq_lens.to(dev)
        pt = None if w.page_table is None else w.page_table.to(dev)
        tp.hadamard_apply(q, LATENT)
        tp.hadamard_apply(cache, LATENT)
        W = None
        if w.W_uv is not None:
            Wt = w.W_uv.to(dev).transpose(1, 2).contiguous()
            tp.hadamard_apply(Wt, LATENT)
            W = Wt.transpose(1, 2).contiguous()
        small = cache.numel() * 2 < 2 * L2_BYTES
        tokens = int(w.seq_lens.to(torch.int64).sum())
        cs = ClockSampler(dev.index or 0)
        cs.start()
        time.sleep(0.2)
        rows = []
        for st in settings:
            G, rope = st["G"], st["rope"]
            out = torch.empty((w.B, w.H, LATENT), dtype=torch.float32, device=dev)
            lse = torch.empty((w.B, w.H, G), dtype=torch.float32, device=dev)
            y = torch.empty((w.B, w.H, 128), dtype=torch.float32, device=dev)
            need = tp.decode_workspace_size(q, cache, seq, pt, G, rope, out, num_splits=st["splits"])
            ws = torch.empty(max(16, need), dtype=torch.uint8, device=dev)

            def dec():
                tp.decode(q, cache, seq, pt, G, rope, w.scale, out=out, lse=lse,
                          num_splits=st["splits"], workspace=ws)

            def timed(fn, n):
                ts = []
                for _ in range(3):
                    fn()
                for i in range(n):
                    if small or i == 0:
                        flush.zero_()
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record()
                    fn()
                    b.record()
                    if small:
                        torch.cuda.synchronize()
                        ts.append(a.elapsed_time(b))
                    else:
                        ts.append((a, b))
                torch.cuda.synchronize()
                if not small:
                    ts = [x.elapsed_time(z) for x, z in ts]
                return statistics.median(ts) / 1e3

            t = timed(dec, 50)
            nb = w.latent_kv_bytes(G, None, rope)
            fl = tokens * w.H * flops_per_token_head(G, None, rope)
            t_roof = max(nb / (hbm_peak * 1e9), fl / (tc_peak * 1e12))
            row = {"G": G, "rope": rope, "splits": st["splits"] or "auto",
                   "decode_us": round(t * 1e6, 1), "GB_s": round(nb / t / 1e9, 1),
                   "hbm_frac": round(nb / t / 1e9 / hbm_peak, 4),
                   "tensor_tflops": round(fl / t / 1e12, 1),
                   "roofline_frac": round(t_roof / t, 4),
                   "tok_s_layer": round(w.B / t, 1)}
            if st["vup"] and W is not None:
                tv = timed(lambda: tp.vup_combine(out, W, y), 50)
                vb = out.numel() * 4 + W.numel() * 2 + y.numel() * 4
                row.update({"vup_us": round(tv * 1e6, 2),
                            "vup_hbm_frac": round(vb / tv / 1e9 / hbm_peak, 4),
                            "step_us": round((t + tv) * 1e6, 1)})
            rows.append(row)
            del out, lse, y, ws
        res[name] = {"B": w.B, "H": w.H, "tokens": tokens,
                     "cache_bytes": int(cache.numel() * 2),
                     "timing": "median of 50 launches, L2 flushed before each" if small
                               else "median of 50 back-to-back launches (cache > 2x L2)",
                     "rows": rows, "clocks": cs.stop()}
        del q, cache, seq, pt, W
        torch.cuda.empty_cache()
    del flush
    return res


def _median_us(fn, n, warm=2):
    for _ in range(warm):
        fn()
    ts = []
    for _ in range(n):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        ts.append((a, b))
    torch.cuda.synchronize()
    return statistics.median([x.elapsed_time(z) for x, z in ts]) * 1e3


def setup_ops(tp, dev, cache, host_cache, hbm_peak):
    """The steps around the decode on the DeepSeek-V3 workload, each the
    median of a few calls timed with CUDA events: the Hadamard rotation of
    the whole stored cache (one-off; an even number of calls leaves it as it
    was), the cache append of one decode step's 64 new rows and of a
    65536-row batch (f32 rows in, Hadamard, two norm groups), and the PCA
    calibration covariance over 262144 unrotated cache rows and the PCA
    rotation of those rows, with the eigenvalue-sum shares of the G = 2 and
    G = 4 shards (Eq. 25's alpha and beta) as information."""
    res = {}
    nb = cache.numel() // WIDTH * LATENT * 2  # the latent columns, read and written once
    t = _median_us(lambda: tp.hadamard_apply(cache, LATENT), 4)
    res["hadamard_cache"] = {"bytes": 2 * nb, "us": round(t, 1),
                             "GB_s": round(2 * nb / t / 1e3, 1),
                             "hbm_frac": round(2 * nb / t / 1e3 / hbm_peak, 4)}
    g = torch.Generator().manual_seed(77)
    for rows in (64, 65536):
        blocks = (rows + 63) // 64
        dst = torch.zeros((blocks, 64, WIDTH), dtype=torch.bfloat16, device=dev)
        new = torch.randn((rows, WIDTH), generator=g).to(dev)
        pt = torch.arange(blocks, dtype=torch.int32, device=dev).repeat_interleave(64)[:rows]
        pt = pt.reshape(rows, 1).contiguous()
        pos = (torch.arange(rows, dtype=torch.int32) % 64).to(dev)
        t = _median_us(lambda: tp.cache_append(new, pos, pt, dst, norm_groups=2, hadamard=True), 20)
        by = rows * WIDTH * (4 + 2)
        res[f"append_{rows}"] = {"rows": rows, "bytes": by, "us": round(t, 2),
                                 "GB_s": round(by / t / 1e3, 1),
                                 "hbm_frac": round(by / t / 1e3 / hbm_peak, 4)}
        del dst, new, pt, pos
    n = 262144
    rows = host_cache.view(-1, WIDTH)[:n].to(dev)
    mean, cov = tp.latent_covariance(rows)
    t = _median_us(lambda: tp.latent_covariance(rows), 5)
    fl = 2.0 * n * LATENT * LATENT
    res["pca_covariance"] = {"rows": n, "us": round(t, 1),
                             "GB_s": round(rows.numel() * 2 / t / 1e3, 1),
                             "fma_tflops": round(fl / t / 1e6, 2)}
    lam, vec = torch.linalg.eigh(cov.double().cpu())
    order = torch.argsort(lam, descending=True)
    lam, vec = lam[order], vec[:, order]
    U = vec.to(torch.bfloat16).contiguous().to(dev)
    t = _median_us(lambda: tp.rotate_apply(rows, U), 5)
    res["pca_rotate"] = {"rows": n, "us": round(t, 1),
                         "GB_s": round(2 * rows.numel() * 2 / t / 1e3, 1)}
    tot = float(lam.sum())
    res["pca_shares"] = {f"G{G}": [round(float(lam[i * (LATENT // G):(i + 1) * (LATENT // G)].sum())
                                         / tot, 4) for i in range(G)] for G in (2, 4)}
    del rows, U
    torch.cuda.empty_cache()
    return res


def prefill_workload(tp, dev, tc_peak):
    """Prefill of one DeepSeek-V3-shaped request (H = 128) under prefill/decode
    separation: the prompt rows into the paged cache, then exact MLA (G = 1)
    of every prompt token over its causal prefix (tpla_prefill).  FLOPs are
    the absorbed form's 2176 per (query token, cached token, head) over the
    causal pairs; the prompt's cache (T x 1152 B) stays in L2, so the bound is
    the tensor pipe.  Median of 10 calls after 3 warm-up calls."""
    from mla_latent_kv_dim_b200.workloads import make_prefill_inputs
    res = {"rows": [], "timing": "median of 10 calls (append + attention + merge)"}
    cs = ClockSampler(dev.index or 0)
    cs.start()
    time.sleep(0.2)
    for T in (4096, 16384):
        w = make_prefill_inputs(T, 128, 0, seed=31)
        q, new = w.q.to(dev), w.kv_new.to(dev)
        row, cache = w.page_row.to(dev), w.cache.to(dev)
        out = torch.empty((T, 128, LATENT), dtype=torch.float32, device=dev)
        lse = torch.empty((T, 128, 1), dtype=torch.float32, device=dev)
        ws = torch.empty(1 << 24, dtype=torch.uint8, device=dev)

        def call():
            tp.prefill(q, new, 0, row, cache, scale=w.scale, out=out, lse=lse, workspace=ws)

        for _ in range(3):
            call()
        ts = []
        for _ in range(10):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        t = statistics.median([x.elapsed_time(z) for x, z in ts]) / 1e3
        pairs = T * (T + 1) // 2
        fl = pairs * 128 * flops_per_token_head(1)
        res["rows"].append({"T": T, "H": 128, "causal_pairs": pairs,
                            "prefill_us": round(t * 1e6, 1),
                            "tensor_tflops": round(fl / t / 1e12, 1),
                            "tensor_frac": round(fl / t / 1e12 / tc_peak, 4),
                            "prompt_tok_s": round(T / t, 1)})
        del q, new, row, cache, out, lse, ws
        torch.cuda.empty_cache()
    res["clocks"] = cs.stop()
    return res


def _sm100_used(tp, q, cache, seq, pt, G, rope, out, args):
    try:
        tp.decode_workspace_size(q, cache, seq, pt, G, rope, out, kernel="sm100")
        return True
    except tp.TplaError:
        return False


def run_profile(args):
    """Decode launches only (for ncu captures): W warm-up + K timed launches.
    With --prefill T: prefill calls of one T-token prompt instead."""
    import mla_latent_kv_dim_b200 as tp
    dev = torch.device("cuda", 0)
    if args.prefill > 0:
        from mla_latent_kv_dim_b200.workloads import make_prefill_inputs
        T = args.prefill
        pw = make_prefill_inputs(T, 128, 0, seed=31)
        q, new, row, cache = pw.q.to(dev), pw.kv_new.to(dev), pw.page_row.to(dev), pw.cache.to(dev)
        out = torch.empty((T, 128, LATENT), dtype=torch.float32, device=dev)
        lse = torch.empty((T, 128, 1), dtype=torch.float32, device=dev)
        ws = torch.empty(1 << 24, dtype=torch.uint8, device=dev)

        def call():
            tp.prefill(q, new, 0, row, cache, scale=pw.scale, out=out, lse=lse, workspace=ws)

        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            call()
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) / 1e3 / args.steps
        fl = T * (T + 1) // 2 * 128 * flops_per_token_head(1)
        print(json.dumps({"profile": "prefill", "T": T, "prefill_us": round(t * 1e6, 1),
                          "tensor_tflops": round(fl / t / 1e12, 1),
                          "status": tp.device_status()}), flush=True)
        return 0
    w = make_workload(args.config, batch=args.batch)
    q, cache, seq = w.q.to(dev), w.cache.to(dev), w.seq_lens.to(dev)
    pt = None if w.page_table is None else w.page_table.to(dev)
    out = torch.empty((w.B, w.H, LATENT), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, w.H, args.G), dtype=torch.float32, device=dev)
    need = tp.decode_workspace_size(q, cache, seq, pt, args.G, args.rope, out,
                                    num_splits=args.num_splits, kernel=args.kernel)
    ws = torch.empty(max(16, need), dtype=torch.uint8, device=dev)

    def once():
        tp.decode(q, cache, seq, pt, args.G, args.rope, w.scale, out=out, lse=lse,
                  num_splits=args.num_splits, kernel=args.kernel, workspace=ws)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        once()
    b.record()
    torch.cuda.synchronize()
    t = a.elapsed_time(b) / 1e3 / args.steps
    nb = w.latent_kv_bytes(args.G)
    print(json.dumps({"profile": args.config, "B": w.B, "G": args.G, "decode_us": round(t * 1e6, 1),
                      "GB_s": round(nb / t / 1e9, 1), "status": tp.device_status()}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.profile:
        return run_profile(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
