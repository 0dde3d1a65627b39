#!/usr/bin/env python
"""Benchmark: latency of one 10-step action chunk of the pi0-class bf16 action
expert (18 layers, width 1024, 8 q / 1 kv heads, head_dim 256, GeGLU 4096,
816-token prefix KV, 1 state + 50 action tokens, batch 1), and the HBM
bandwidth it achieves.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --workload flash-draft      # the FLASH draft model alone
    python bench.py --workload gemma2b-prefill  # VLM prefill + the pi0-bf16 chunk, one graph

One "step" is one call of rtv_denoise: the whole hot path (10 Euler steps
through the expert) over one batch of synthetic input.  With N > 1 the
script is launched by torchrun, one process per GPU; every rank runs an
independent replica (weak scaling, no data-path collective) and the time is
the max over ranks.  Rank 0 prints one JSON line.

Timing: W untimed warm-up calls, then K calls bracketed by a barrier and a
device synchronise, timed with CUDA events on the launching stream.  The
expert's 623 MB of weights stream from HBM on every step (L2 is 126 MB), so
no separate L2 flush is done.  `e2e` repeats the measurement through the C
ABI with pinned host buffers, the host<->device copies inside the timed
region.  `cpu_baseline` times the CPU oracle on a bounded sample.
"""

from __future__ import annotations

import argparse
import glob
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

METRIC = "10-step action-chunk latency (us) and achieved HBM GB/s vs 8 TB/s roofline"
PREFILL_METRIC = ("prefill + 10-step chunk latency (us): Gemma-2B-class prefill over 816 tokens writing the "
                  "KV cache, then the pi0-bf16 chunk, one CUDA graph")
DRAFT_METRIC = "FLASH draft forward latency (us): one Gemma-2B-width block + action head over 768 image tokens"
# Earlier measurements on this machine's B200s, used only when MEASURED_PEAKS.json is absent: a STREAM-style
# copy, and a cuBLAS bf16 GEMM as a burst and as a seconds-long loop under the power cap.
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="pi0-bf16")
    ap.add_argument("--n-steps", type=int, default=10, help="Euler steps per chunk")
    ap.add_argument("--batch", type=int, default=0,
                    help="independent chunks per call, each with its own prefix (default: the workload's)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (profiling runs on smaller captures only; "
                         "the JSON line then names the reduced depth)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-round", action="store_true",
                    help="skip the FLASH draft model / dual-path round measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU seconds of the oracle sample")
    ap.add_argument("--trace", action="store_true",
                    help="print the library's phase stamps of layer 0 of the first Euler step (no timing)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------

def algorithmic_bytes_per_step(cfg, batch=1):
    """Weight bytes of every layer and of the state/action projections, plus
    the prefix K and V of every layer, each counted once per Euler step.
    The time MLP depends only on t and is precomputed, so it is excluded, and
    so are the per-layer time modulator's weights (its rows and shift terms
    are tables of the Euler schedule); Pi0's concat time MLP reads its
    action half (w x w) and output layer (w x w) every step."""
    elt = 4 if cfg.dtype == "f32" else 2
    w, f = cfg.width, cfg.mlp_dim
    mlp_elt = 1 if cfg.mlp_dtype == "fp8_e4m3" else elt
    attn = w * (cfg.q_dim + 2 * cfg.kv_dim) + cfg.q_dim * w
    layer = attn * elt + 3 * w * f * mlp_elt
    proj = (w * cfg.state_dim + w * cfg.action_dim + cfg.action_dim * w) * elt
    if getattr(cfg, "time_cond", "add") == "concat":
        proj += 2 * w * w * elt
    kv = 2 * batch * cfg.prefix_len * cfg.kv_dim * elt
    return cfg.n_layers * (layer + kv) + proj


# DRAM bytes (read + written) of one pi0-bf16 chunk (18 layers, P = 816, batch 1), summed by ncu over the 911
# launches of a chunk with the L2 carried between kernels (profiles/dram_traffic_pi0-bf16_full_depth.md).  The
# figure holds for the kernel sources it was taken on, identified by their SHA-256; after any change to them the
# bench reports null until the capture is taken again.
TRAFFIC_PI0_BF16 = {"bytes_per_chunk": 6436925184,
                    "kernel_sources_sha256": "c2d3101a5c66b9f059bae20464169b3afb1e7a8780188a8b1b2f640ec3843f1e"}


def kernel_sources_sha256():
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "flow_matching_action_dm0_b200", "csrc", "*"))):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(os.path.basename(f).encode())
            with open(f, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------
# clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step_seconds_threads(cfg, target_s: float, threads=None, min_samples: int = 5, max_samples: int = 10):
    """oracle_step_seconds with the BLAS thread pool limited to `threads`
    (None: as configured, i.e. every host core)."""
    if threads is None:
        return oracle_step_seconds(cfg, target_s, min_samples, max_samples)
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None, 0
    with threadpool_limits(limits=threads, user_api="blas"):
        return oracle_step_seconds(cfg, target_s, min_samples, max_samples)


def oracle_step_seconds(cfg, target_s: float, min_samples: int = 5, max_samples: int = 10):
    """Seconds per Euler step of the CPU oracle on the workload (bounded
    sample: median of at least min_samples steps)."""
    from oracle import expert as O
    from synthetic import make_noise, make_prefix_kv, make_state, make_weights
    W = O.to_f64(make_weights(cfg))
    kv = make_prefix_kv(cfg)
    x = make_noise(cfg)[0].astype(np.float64)
    state = make_state(cfg)[0]
    pk, pv = kv[:, 0, 0].astype(np.float64), kv[:, 1, 0].astype(np.float64)
    times = []
    t_total = 0.0
    k = 0
    while (k < min_samples or t_total < target_s) and k < max_samples:
        t = 1.0 - (k % cfg.n_steps) / cfg.n_steps
        t0 = time.perf_counter()
        v = O.expert_velocity(W, cfg, x, state, t, pk, pv)
        x = x - v / cfg.n_steps
        dt = time.perf_counter() - t0
        times.append(dt)
        t_total += dt
        k += 1
    return statistics.median(times), k


def run_reference_draft(args, info):
    """The CPU oracle's draft forward on the flash-draft workload: each step
    is one whole forward (about 110M parameters x 818 rows in fp64)."""
    from oracle import draft as OD
    from synthetic import get_draft_config, make_draft_weights, make_visual_tokens
    dcfg = get_draft_config(args.workload)
    W = make_draft_weights(dcfg)
    vis = make_visual_tokens(dcfg)[0]
    steps = max(1, min(args.steps, 3))
    OD.draft_forward(W, dcfg, vis)
    t0 = time.perf_counter()
    for _ in range(steps):
        OD.draft_forward(W, dcfg, vis)
    us = (time.perf_counter() - t0) / steps * 1e6
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": DRAFT_METRIC, "value": us, "unit": "us", "n_gpus": args.gpus,
        "steps": steps, "warmup": 1, "ms_per_step": us / 1000.0, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "n_vis": dcfg.n_vis, "n_queries": dcfg.n_queries, "batch": 1},
        "cpu_baseline": {"value": us, "unit": "us", "cores": cores, "kind": "oracle",
                         "sample": f"{steps} whole draft forwards (fp64 numpy oracle)"},
        "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_prefill(args, info):
    """The CPU oracle on the gemma2b-prefill workload, bounded: each step is a
    2-layer oracle prefill over the 816 tokens (one full layer and the last
    layer's K/V, weight generation included) scaled to the stack's depth,
    plus one oracle Euler step of the pi0-bf16 expert scaled to the chunk."""
    from oracle import expert as O
    from oracle import prefill as OP
    from synthetic import (get_config, get_prefill_config, make_noise, make_prefill_weights, make_prefix_embeddings,
                           make_prefix_kv, make_state, make_weights)
    pc = get_prefill_config(args.workload)
    cfg = get_config("pi0-bf16", n_steps=args.n_steps, prefix_len=pc.n_tokens)
    two = pc.with_(n_layers=2)
    emb = make_prefix_embeddings(pc)
    W = O.to_f64(make_weights(cfg))
    kv = make_prefix_kv(cfg)
    pk, pv = kv[:, 0, 0].astype(np.float64), kv[:, 1, 0].astype(np.float64)
    x = make_noise(cfg)[0].astype(np.float64)
    state = make_state(cfg)[0]
    steps = max(1, min(args.steps, 2))
    t0 = time.perf_counter()
    for _ in range(steps):
        OP.prefill_kv(lambda l: make_prefill_weights(two, layers=[l]), two, emb)
    t_pre = (time.perf_counter() - t0) / steps
    t0 = time.perf_counter()
    O.expert_velocity(W, cfg, x, state, 1.0, pk, pv)
    t_step = time.perf_counter() - t0
    us = (t_pre * (pc.n_layers - 1) + t_step * cfg.n_steps) * 1e6
    line = {
        "impl": "reference", "metric": PREFILL_METRIC, "value": us, "unit": "us", "n_gpus": args.gpus,
        "steps": steps, "warmup": 0, "ms_per_step": us / 1000.0, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "n_tokens": pc.n_tokens, "expert": "pi0-bf16", "n_steps": cfg.n_steps},
        "cpu_baseline": {"value": us, "unit": "us", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{steps} 2-layer oracle prefills scaled to {pc.n_layers} layers + one oracle "
                                   f"Euler step scaled x{cfg.n_steps}"},
        "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference(args, info):
    """The CPU oracle, as it stands, on a bounded sample of the workload:
    each step is one Euler step of the chunk, scaled to chunk latency."""
    if not info.is_main:
        return
    from synthetic import DRAFTS, PREFILLS
    if args.workload in DRAFTS:
        run_reference_draft(args, info)
        return
    if args.workload in PREFILLS:
        run_reference_prefill(args, info)
        return
    from synthetic import get_config
    cfg = get_config(args.workload, n_steps=args.n_steps)
    from oracle import expert as O
    from synthetic import make_noise, make_prefix_kv, make_state, make_weights
    W = O.to_f64(make_weights(cfg))
    kv = make_prefix_kv(cfg)
    pk, pv = kv[:, 0, 0].astype(np.float64), kv[:, 1, 0].astype(np.float64)
    x = make_noise(cfg)[0].astype(np.float64)
    state = make_state(cfg)[0]
    for _ in range(max(0, min(args.warmup, 1))):
        O.expert_velocity(W, cfg, x, state, 1.0, pk, pv)
    steps = max(1, min(args.steps, 20))
    t0 = time.perf_counter()
    for k in range(steps):
        t = 1.0 - (k % cfg.n_steps) / cfg.n_steps
        x = x - O.expert_velocity(W, cfg, x, state, t, pk, pv) / cfg.n_steps
    per_step = (time.perf_counter() - t0) / steps
    chunk_us = per_step * cfg.n_steps * 1e6
    cores = blas_threads()
    # one timed step is one Euler step of the chunk: steps x ms_per_step is the
    # time actually spent; value is that per-step time scaled to a whole chunk
    line = {
        "impl": "reference", "metric": METRIC, "value": chunk_us, "unit": "us", "n_gpus": args.gpus,
        "steps": steps, "warmup": min(args.warmup, 1), "ms_per_step": per_step * 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "n_steps": cfg.n_steps, "batch": 1, "prefix_len": cfg.prefix_len,
                   "layers": cfg.n_layers, "width": cfg.width, "path": "cpu oracle (fp64 numpy)",
                   "step": f"one Euler step of the chunk; value = ms_per_step x {cfg.n_steps} (chunk latency)"},
        "cpu_baseline": {"value": chunk_us, "unit": "us", "cores": cores, "kind": "oracle",
                         "sample": f"{steps} single Euler steps of the {args.workload} chunk (fp64 numpy oracle), "
                                   f"mean scaled x{cfg.n_steps} to chunk latency"},
        "e2e": {"value": chunk_us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, info):
    import torch

    from flow_matching_action_dm0_b200 import ActionExpert
    from flow_matching_action_dm0_b200 import replicas as R
    from synthetic import (f32_to_bf16_bits, get_config, make_draft, make_noise, make_prefix_kv, make_state,
                           make_weights)

    dev = info.local_rank
    torch.cuda.set_device(dev)
    cfg = get_config(args.workload, n_steps=args.n_steps)
    if args.layers > 0:
        cfg = cfg.with_(n_layers=args.layers)
    if args.batch > 0:
        cfg = cfg.with_(batch=args.batch)
    weights = make_weights(cfg)
    kv = make_prefix_kv(cfg)
    noise = make_noise(cfg)
    state = make_state(cfg)

    ex = ActionExpert(cfg, device=dev, max_batch=cfg.batch, max_taus=4)
    ex.load(weights)
    del weights
    if cfg.dtype == "bf16":
        kv_t = torch.from_numpy(f32_to_bf16_bits(kv).view(np.int16)).view(torch.bfloat16).cuda(dev)
    else:
        kv_t = torch.from_numpy(kv).cuda(dev)
    stream = torch.cuda.Stream(dev)
    ex.set_prefix_kv(kv_t, stream=stream)
    noise_d = torch.from_numpy(noise).cuda(dev)
    state_d = torch.from_numpy(state).cuda(dev)
    out_d = torch.empty_like(noise_d)
    torch.cuda.synchronize(dev)

    n = cfg.n_steps
    for _ in range(max(3, args.warmup)):
        ex.denoise(noise_d, state_d, n, out_d, stream=stream)
    torch.cuda.synchronize(dev)
    s, bits = ex.status()
    if s != 0:
        raise RuntimeError(f"device status {bits:#x} after warm-up")

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    R.barrier(info, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for _ in range(K):
            ex.denoise(noise_d, state_d, n, out_d, stream=stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    R.barrier(info, dev)
    ms_local = start.elapsed_time(end) / K
    ms = R.max_over_ranks(ms_local, info, dev)
    s, bits = ex.status()
    if s != 0:
        raise RuntimeError(f"device status {bits:#x} after the timed region")

    # latency distribution: each call bracketed by its own events and waited
    # for (no overlap between calls), at least 50 calls
    lat = []
    for _ in range(max(50, K)):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        ex.denoise(noise_d, state_d, n, out_d, stream=stream)
        c1.record(stream)
        c1.synchronize()
        lat.append(c0.elapsed_time(c1) * 1000.0)
    lat = np.asarray(lat)
    latency = {"unit": "us", "calls": int(lat.size), "p50": float(np.percentile(lat, 50)),
               "p90": float(np.percentile(lat, 90)), "p99": float(np.percentile(lat, 99)),
               "mean": float(lat.mean()), "min": float(lat.min()), "max": float(lat.max()),
               "note": "per-call CUDA events on the launching stream, each call waited for before the next"}

    # end to end through the C ABI with pinned host buffers
    noise_h = torch.from_numpy(noise).pin_memory()
    state_h = torch.from_numpy(state).pin_memory()
    out_h = torch.empty_like(noise_h).pin_memory()
    for _ in range(2):
        ex.denoise(noise_h, state_h, n, out_h, stream=stream)
    torch.cuda.synchronize(dev)
    R.barrier(info, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        ex.denoise(noise_h, state_h, n, out_h, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    R.barrier(info, dev)
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1) / K, info, dev)

    # FLASH verification of one draft chunk at the workload's taus: one expert
    # evaluation of len(taus) suffixes plus the decision, host buffers in and
    # out (the call waits for its result); device time per call, median
    draft = make_draft(cfg)
    taus = tuple(cfg.taus)
    for _ in range(3):
        ex.verify(draft, noise, state, taus, 0.05, cfg.gripper, want_dist=False, stream=stream)
    v_ms = []
    for _ in range(max(5, min(K, 20))):
        v0, v1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        v0.record(stream)
        ex.verify(draft, noise, state, taus, 0.05, cfg.gripper, want_dist=False, stream=stream)
        v1.record(stream)
        torch.cuda.synchronize(dev)
        v_ms.append(v0.elapsed_time(v1))
    verify_us = float(np.median(v_ms)) * 1000.0

    round_info = None
    if info.world == 1 and not args.no_round and cfg.batch == 1 and args.layers <= 0 and \
            (cfg.chunk_len, cfg.action_dim) == (50, 32):
        round_info = measure_round(ex, cfg, noise_d, state_d, stream, dev, K)

    launches_per_call = ex.kernels_per_call(n)
    path = ex.path
    ex.close()

    if not info.is_main:
        return
    peaks, peak_kind = load_peaks()
    bytes_step = algorithmic_bytes_per_step(cfg, batch=cfg.batch)
    bytes_chunk = bytes_step * n
    achieved = bytes_chunk / (ms * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])
    traffic, traffic_note = None, "DRAM bytes were captured for pi0-bf16 at full depth only"
    if args.workload == "pi0-bf16" and args.layers <= 0 and n == 10 and cfg.batch == 1:
        if kernel_sources_sha256() == TRAFFIC_PI0_BF16["kernel_sources_sha256"]:
            traffic = TRAFFIC_PI0_BF16["bytes_per_chunk"]
            traffic_note = ("ncu dram__bytes_read.sum + dram__bytes_write.sum over the 911 launches of one chunk, "
                            "L2 carried between kernels; bytes per chunk (traffic / algorithmic = "
                            f"{traffic / bytes_chunk:.3f})")
        else:
            traffic_note = "the kernel sources changed since the DRAM capture: not yet taken again"
    line = {
        "metric": METRIC,
        "value": ms * 1000.0,
        "unit": "us",
        "n_gpus": info.world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic",
        "config": {"workload": args.workload if args.layers <= 0 else f"{args.workload} ({cfg.n_layers} layers)",
                   "n_steps": n, "batch": cfg.batch, "prefix_len": cfg.prefix_len,
                   "layers": cfg.n_layers, "width": cfg.width, "parallelism": f"replicas x{info.world}",
                   "l2": "inputs larger than L2: 623 MB of weights stream from HBM every Euler step; no flush",
                   "path": path},
        "chunks_per_s": info.world * cfg.batch * 1000.0 / ms,
        "roofline": {"bound": "hbm", "kernel": "whole denoise graph (all kernels of one chunk)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} hbm_gbs", "algorithmic_bytes_per_launch": bytes_chunk,
                     "traffic": traffic,
                     "traffic_note": traffic_note},
        "e2e": {"value": e2e_ms * 1000.0, "unit": "us",
                "h2d_bytes_per_step": int(noise.nbytes + state.nbytes), "d2h_bytes_per_step": int(noise.nbytes)},
        "latency": latency,
        "clocks": clk.summary(),
        "gpu_launches": int(launches_per_call * K) if launches_per_call > 0 else None,
        "verify": {"taus": list(taus), "us_per_call": verify_us,
                   "ratio_to_one_euler_step": verify_us / (ms * 1000.0 / n),
                   "note": "one FLASH verification (len(taus) suffixes in one expert evaluation + decision), "
                           "host buffers, device time per call (median)"},
    }
    if round_info is not None:
        line["flash_round"] = round_info
    if info.world == 1 and not args.no_cpu_baseline:
        per_step_s, k = oracle_step_seconds_threads(cfg, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": per_step_s * n * 1e6, "unit": "us", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{k} single Euler steps of the {args.workload} chunk (fp64 numpy oracle, median), "
                      f"scaled x{n} to one chunk; BLAS threads = host cores"}
        one_s, k1 = oracle_step_seconds_threads(cfg, args.cpu_seconds / 2, threads=1)
        if one_s is not None:
            line["cpu_baseline"]["single_thread"] = {
                "value": one_s * n * 1e6, "unit": "us", "cores": 1,
                "sample": f"{k1} single Euler steps, median, scaled x{n}; BLAS limited to one thread"}
    print(json.dumps(line), flush=True)


def draft_bytes(dcfg) -> int:
    """Algorithmic bytes of one draft forward: the block's and head's weights,
    the queries' residual rows, the image features read, and their keys/values
    written and read back once.  On the tensor-core path (bf16) the action
    queries' q/k/v depend on the weights only and are computed once per graph:
    a forward reads their tiles instead of the q projection's weights."""
    e = 2 if dcfg.dtype == "bf16" else 4
    w = dcfg.width
    kv = dcfg.n_vis * 2 * dcfg.kv_dim * e
    total = (dcfg.block_params() - 2 * w) * e + 2 * w * 4 + dcfg.action_dim * (w * e + 4) + \
        dcfg.n_queries * w * 4 + dcfg.n_vis * w * e + 2 * kv
    if dcfg.dtype == "bf16":
        folded_tiles = (dcfg.n_q_heads // 2) * 128 * dcfg.head_dim * 2 + 2 * dcfg.n_kv_heads * 64 * dcfg.head_dim * 2
        total += folded_tiles - w * dcfg.q_dim * e
    return total


def measure_round(ex, cfg, noise, state, stream, dev, K):
    """FLASH draft model (the flash-draft workload: one Gemma-2B-width block,
    110M parameters, 768 image tokens) and one dual-path round on the
    expert: device time of the draft forward, and of a whole round in each
    branch (CUDA events around the call; the host reads the verdict in
    between, so the span includes that gap)."""
    import torch

    from flow_matching_action_dm0_b200 import DraftModel, flash_round
    from synthetic import f32_to_bf16_bits, get_draft_config, make_draft_weights, make_visual_tokens

    dcfg = get_draft_config("flash-draft")
    dw = make_draft_weights(dcfg)
    # accept branch: the head's gripper row is zeroed and its bias made
    # positive, so the random draft holds the gripper still (no switch)
    dw_acc = dict(dw)
    dw_acc["action_head.w"] = dw["action_head.w"].copy()
    dw_acc["action_head.w"][cfg.gripper] = 0.0
    dw_acc["action_head.b"] = dw["action_head.b"].copy()
    dw_acc["action_head.b"][cfg.gripper] = 0.5
    vis = make_visual_tokens(dcfg)
    vis_d = torch.from_numpy(f32_to_bf16_bits(vis).view(np.int16)).view(torch.bfloat16).cuda(dev)
    out_d = torch.empty((1, dcfg.n_queries, dcfg.action_dim), dtype=torch.float32, device=dev)
    taus = tuple(cfg.taus)
    res = {"draft_workload": "flash-draft", "draft_params": dcfg.params(), "n_vis": dcfg.n_vis, "taus": list(taus),
           "n_steps": cfg.n_steps}
    for branch, weights, delta in (("accept", dw_acc, 1e6), ("fallback", dw, 0.05)):
        dm = DraftModel(dcfg, device=dev, max_batch=1)
        dm.load(weights)
        for _ in range(3):
            dm.forward(vis_d, out_d, stream=stream)
        torch.cuda.synchronize(dev)
        if branch == "accept":
            d_ms = []
            for _ in range(max(10, min(K, 50))):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                dm.forward(vis_d, out_d, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                d_ms.append(e0.elapsed_time(e1))
            draft_us = float(np.median(d_ms)) * 1000.0
            nbytes = draft_bytes(dcfg)
            res["draft_us"] = draft_us
            res["draft_kernels"] = dm.kernels_per_call(dcfg.n_vis, 1)
            res["draft_roofline"] = {"bound": "hbm", "algorithmic_bytes": nbytes,
                                     "achieved": nbytes / (draft_us * 1e-6) / 1e9, "unit": "GB/s"}
        r = None
        for _ in range(2):
            r = flash_round(ex, dm, vis_d[0], noise[0], state[0], taus, delta, cfg.gripper, cfg.n_steps,
                            stream=stream)
        r_ms = []
        for _ in range(max(5, min(K, 20))):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            r = flash_round(ex, dm, vis_d[0], noise[0], state[0], taus, delta, cfg.gripper, cfg.n_steps,
                            stream=stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            r_ms.append(e0.elapsed_time(e1))
        res[f"round_{branch}_us"] = float(np.median(r_ms)) * 1000.0
        res[f"round_{branch}_verdict"] = {"accepted_len": r.accepted_len, "flags": r.flags,
                                          "used_full": r.used_full, "delta": delta}
        s, bits = dm.status()
        if s != 0:
            raise RuntimeError(f"draft device status {bits:#x}")
        dm.close()
    res["note"] = ("accept branch = draft + verify + verdict read + draft copied out (gripper row of the random "
                   "head zeroed, bias 0.5, delta 1e6); fallback branch = the same + 10-step denoise (random head, "
                   "gripper switches); device time per round, median, CUDA events around the synchronous call")
    return res


def run_draft(args, info):
    """The FLASH draft model alone (workload flash-draft): one step is one
    rtv_draft_forward over one observation's 768 image tokens."""
    import torch

    from flow_matching_action_dm0_b200 import DraftModel
    from flow_matching_action_dm0_b200 import replicas as R
    from synthetic import f32_to_bf16_bits, get_draft_config, make_draft_weights, make_visual_tokens

    dev = info.local_rank
    torch.cuda.set_device(dev)
    dcfg = get_draft_config(args.workload)
    if args.batch > 0:
        dcfg = dcfg.with_(batch=args.batch)
    B = dcfg.batch
    vis = make_visual_tokens(dcfg)
    dm = DraftModel(dcfg, device=dev, max_batch=B)
    dm.load(make_draft_weights(dcfg))
    bits = f32_to_bf16_bits(vis).view(np.int16) if dcfg.dtype == "bf16" else vis
    vis_t = torch.from_numpy(bits)
    if dcfg.dtype == "bf16":
        vis_t = vis_t.view(torch.bfloat16)
    vis_d = vis_t.cuda(dev)
    out_d = torch.empty((B, dcfg.n_queries, dcfg.action_dim), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    for _ in range(max(3, args.warmup)):
        dm.forward(vis_d, out_d, stream=stream)
    torch.cuda.synchronize(dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    R.barrier(info, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for _ in range(K):
            dm.forward(vis_d, out_d, stream=stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    R.barrier(info, dev)
    ms = R.max_over_ranks(start.elapsed_time(end) / K, info, dev)
    s, bits_ = dm.status()
    if s != 0:
        raise RuntimeError(f"device status {bits_:#x} after the timed region")
    vis_h = vis_t.pin_memory()
    out_h = torch.empty_like(out_d, device="cpu").pin_memory()
    for _ in range(2):
        dm.forward(vis_h, out_h, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        dm.forward(vis_h, out_h, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1) / K, info, dev)
    kernels = dm.kernels_per_call(dcfg.n_vis, B)
    path = dm.path
    dm.close()
    if not info.is_main:
        return
    peaks, peak_kind = load_peaks()
    nbytes = draft_bytes(dcfg) + (B - 1) * (dcfg.n_vis * dcfg.width * 2 + dcfg.n_vis * 4 * dcfg.kv_dim)
    achieved = nbytes / (ms * 1e-3) / 1e9
    peak = float(peaks["hbm_gbs"])
    line = {
        "metric": DRAFT_METRIC, "value": ms * 1000.0, "unit": "us", "n_gpus": info.world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": dcfg.dtype, "data": "synthetic",
        "config": {"workload": args.workload, "n_vis": dcfg.n_vis, "n_queries": dcfg.n_queries, "batch": B,
                   "width": dcfg.width, "mlp_dim": dcfg.mlp_dim, "params": dcfg.params(),
                   "parallelism": f"replicas x{info.world}",
                   "l2": "inputs larger than L2: 220 MB of block weights stream from HBM every call; no flush",
                   "path": path},
        "roofline": {"bound": "hbm", "kernel": "whole draft graph", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": nbytes, "traffic": None},
        "e2e": {"value": e2e_ms * 1000.0, "unit": "us", "h2d_bytes_per_step": int(vis_t.numel() * vis_t.element_size()),
                "d2h_bytes_per_step": int(out_d.numel() * 4)},
        "clocks": clk.summary(),
        "gpu_launches": int(kernels * K) if kernels > 0 else None,
    }
    if info.world == 1 and not args.no_cpu_baseline:
        from oracle import draft as OD
        W = make_draft_weights(dcfg)
        t0 = time.perf_counter()
        OD.draft_forward(W, dcfg, vis[0])
        per = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": per * B * 1e6, "unit": "us", "cores": blas_threads(), "kind": "oracle",
                                "sample": "one whole draft forward of one observation (fp64 numpy oracle)"
                                          + (f", x{B} for the batch" if B > 1 else "")}
    print(json.dumps(line), flush=True)


def prefill_weights_bits(pc):
    """The stack's parameters with matrices as bf16 bits, one layer at a time."""
    from synthetic import f32_to_bf16_bits, make_prefill_weights
    out = {}
    for l in range(pc.n_layers):
        for k, v in make_prefill_weights(pc, layers=[l]).items():
            out[k] = f32_to_bf16_bits(v) if v.ndim == 2 else v
    return out


def run_prefill(args, info):
    """Gemma-2B-class prefill over 816 embedding tokens writing the pi0-bf16
    expert's KV cache, then its 10-step chunk, as one CUDA graph (one step =
    one rtv_prefill_denoise).  Also times the prefill alone (rtv_prefill_kv)
    for its tensor-pipe roofline."""
    import torch

    from flow_matching_action_dm0_b200 import ActionExpert, PrefillStack
    from flow_matching_action_dm0_b200 import replicas as R
    from synthetic import (f32_to_bf16_bits, get_config, get_prefill_config, make_noise, make_prefix_embeddings,
                           make_state, make_weights)

    dev = info.local_rank
    torch.cuda.set_device(dev)
    pc = get_prefill_config(args.workload)
    cfg = get_config("pi0-bf16", n_steps=args.n_steps, prefix_len=pc.n_tokens)
    if args.layers > 0:
        pc = pc.with_(n_layers=args.layers)
        cfg = cfg.with_(n_layers=args.layers)
    n = cfg.n_steps
    ex = ActionExpert(cfg, device=dev, max_batch=1, max_taus=4)
    ex.load(make_weights(cfg))
    pf = PrefillStack(pc, device=dev)
    pf.load(prefill_weights_bits(pc))
    emb = make_prefix_embeddings(pc)
    emb_t = torch.from_numpy(f32_to_bf16_bits(emb).view(np.int16)).view(torch.bfloat16)
    emb_d = emb_t.cuda(dev)
    noise, state = make_noise(cfg)[0], make_state(cfg)[0]
    noise_d, state_d = torch.from_numpy(noise).cuda(dev), torch.from_numpy(state).cuda(dev)
    out_d = torch.empty_like(noise_d)
    stream = torch.cuda.Stream(dev)
    for _ in range(max(3, args.warmup)):
        pf.denoise(ex, emb_d, noise_d, state_d, n, out_d, stream=stream)
        pf.kv(ex, emb_d, stream=stream)
    torch.cuda.synchronize(dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    R.barrier(info, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk:
        start.record(stream)
        for _ in range(K):
            pf.denoise(ex, emb_d, noise_d, state_d, n, out_d, stream=stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    R.barrier(info, dev)
    ms = R.max_over_ranks(start.elapsed_time(end) / K, info, dev)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(K):
        pf.kv(ex, emb_d, stream=stream)
    p1.record(stream)
    torch.cuda.synchronize(dev)
    prefill_ms = R.max_over_ranks(p0.elapsed_time(p1) / K, info, dev)
    for h in (pf, ex):
        s, bits = h.status()
        if s != 0:
            raise RuntimeError(f"device status {bits:#x} after the timed region")
    emb_h = emb_t.pin_memory()
    noise_h = torch.from_numpy(noise).pin_memory()
    state_h = torch.from_numpy(state).pin_memory()
    out_h = torch.empty_like(noise_h).pin_memory()
    pf.denoise(ex, emb_h, noise_h, state_h, n, out_h, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        pf.denoise(ex, emb_h, noise_h, state_h, n, out_h, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1) / K, info, dev)
    kernels = pf.kernels_per_call(pc.n_tokens, n)
    pf.close()
    ex.close()
    if not info.is_main:
        return
    peaks, peak_kind = load_peaks()
    flops = pc.flops()
    achieved = flops / (prefill_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    line = {
        "metric": PREFILL_METRIC, "value": ms * 1000.0, "unit": "us", "n_gpus": info.world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload if args.layers <= 0 else f"{args.workload} ({pc.n_layers} layers)",
                   "n_tokens": pc.n_tokens, "prefill_layers": pc.n_layers, "prefill_width": pc.width,
                   "prefill_mlp": pc.mlp_dim, "expert": "pi0-bf16", "n_steps": n, "batch": 1,
                   "parallelism": f"replicas x{info.world}",
                   "l2": "inputs larger than L2: 3.7 GB of stack weights and 623 MB of expert weights per call; "
                         "no flush"},
        "prefill_us": prefill_ms * 1000.0,
        "roofline": {"bound": "tensor", "kernel": "whole prefill graph (rtv_prefill_kv)", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{peak_kind} bf16_tflops_sustained", "algorithmic_flops_per_launch": flops,
                     "traffic": None},
        "e2e": {"value": e2e_ms * 1000.0, "unit": "us",
                "h2d_bytes_per_step": int(emb_t.numel() * 2 + noise.nbytes + state.nbytes),
                "d2h_bytes_per_step": int(noise.nbytes)},
        "clocks": clk.summary(),
        "gpu_launches": int(kernels * K) if kernels > 0 else None,
    }
    if info.world == 1 and not args.no_cpu_baseline:
        from oracle import expert as O
        from oracle import prefill as OP
        from synthetic import make_prefill_weights
        one = pc.with_(n_layers=2)
        t0 = time.perf_counter()
        OP.prefill_kv(lambda l: make_prefill_weights(one, layers=[l]), one, emb)
        t_two = time.perf_counter() - t0
        per_step_s, k = oracle_step_seconds(cfg, args.cpu_seconds / 2)
        line["cpu_baseline"] = {
            "value": (t_two * (pc.n_layers - 1) + per_step_s * n) * 1e6, "unit": "us", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"a 2-layer oracle prefill over {pc.n_tokens} tokens (one full layer + one K/V layer, "
                      f"weight generation included) scaled to {pc.n_layers} layers, plus {k} oracle Euler steps "
                      f"scaled x{n}"}
    print(json.dumps(line), flush=True)


def run_trace(args):
    """One traced chunk: the library prints per-CTA phase stamps (globaltimer)
    of the projections and the attention of layer 0, first Euler step."""
    os.environ["RTV_TRACE"] = "1"
    from flow_matching_action_dm0_b200 import ActionExpert
    from synthetic import get_config, make_noise, make_prefix_kv, make_state, make_weights
    cfg = get_config(args.workload, n_steps=args.n_steps)
    ex = ActionExpert(cfg, max_batch=cfg.batch, max_taus=4)
    ex.load(make_weights(cfg))
    ex.set_prefix_kv(make_prefix_kv(cfg))
    noise, state = make_noise(cfg), make_state(cfg)
    for _ in range(max(3, args.warmup)):
        ex.denoise(noise, state, cfg.n_steps)
    ex.close()


def main(argv=None):
    args = parse_args(argv)
    if args.trace:
        run_trace(args)
        return 0
    from flow_matching_action_dm0_b200 import replicas as R
    info = R.rank_info()
    if args.impl == "reference":
        if info.world > 1 and not info.is_main:
            return 0
        run_reference(args, info)
        return 0
    info = R.init("nccl" if info.world > 1 else "gloo")
    from synthetic import DRAFTS, PREFILLS
    try:
        if args.workload in DRAFTS:
            run_draft(args, info)
        elif args.workload in PREFILLS:
            run_prefill(args, info)
        else:
            run_ours(args, info)
    finally:
        R.shutdown(info)
    return 0


if __name__ == "__main__":
    sys.exit(main())
