"""Benchmark of the MOSS-Image DiT denoising step on B200.

A bench "step" is one denoising step of the 1024^2 sampling loop: the DiT twice (CFG
batch 2: conditional branch, unconditional branch skipping layer 22 inside the slg window
[0.01, 1.0]), then the FP32 CFG combine and the shift-5 flow-matching Euler update.  The
timed steps walk the 50-step schedule from step 0, so the default --steps 50 times one
whole image.  Model: 42 blocks, hidden 3072, 24 heads of 128, FFN 8192, random N(0, 0.02)
BF16 weights (seed 2); 512 synthetic text tokens per branch; latent noise from seed 42.

Prints one JSON line (rank 0).  `value` is DiT forwards/s over all ranks (two forwards per
step); replicas only: each rank runs its own image, no collective on the data path.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DiT forwards/s and s/image at 1024² (50 steps, CFG 3); % BF16 TC peak"
UNIT = "forwards/s"
HEIGHT = WIDTH = 1024
N_TXT = 512
STEPS_PER_IMAGE = 50
CFG, SHIFT, SKIP, SLG = 3.0, 5.0, (22,), (0.01, 1.0)
WORKLOAD = ("1024^2 denoising step of the 42-block DiT (hidden 3072, 24x128 heads, FFN 8192): "
            "4096 image + 512 text tokens per branch, CFG batch 2, uncond skips layer 22 in slg [0.01, 1.0], "
            "steps walk the 50-step shift-5 schedule")


def flops_per_branch_layer(N, D=3072, F=8192):
    """Algorithmic FLOPs of one block on one branch of N tokens, by kernel class."""
    return {
        "gemm_qkv": 2.0 * N * D * 3 * D,
        "attention": 4.0 * N * N * D,
        "gemm_oproj": 2.0 * N * D * D,
        "gemm_gateup": 2.0 * N * D * 2 * F,
        "gemm_down": 2.0 * N * F * D,
    }


def _slg_on(step, steps, a, b):
    p = step / steps
    return a <= p <= b


def step_branch_layers(step, L=42):
    return 2 * L - (len(SKIP) if _slg_on(step % STEPS_PER_IMAGE, STEPS_PER_IMAGE, *SLG) else 0)


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """The largest `value` over all ranks (the device time of the slowest rank); the input
    itself when no process group is initialised."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(steps: int, world: int, ms: float, forwards_per_step: int = 2):
    """Whole-job DiT forwards/s and ms per step: every rank runs `steps` denoising steps of
    its own image (two forwards each), timed as the max over ranks, `ms` in total."""
    forwards = forwards_per_step * steps * world
    return forwards / (ms / 1e3), ms / steps


def kernel_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None when the record
    is missing or the kernel's sources have changed since the counters were taken."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "kernel_traffic.json")))[kernel]
        h = hashlib.sha256()
        for f in rec["sources"]:
            h.update(open(os.path.join(ROOT, f), "rb").read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons, watts = [], 0.0, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            try:
                watts.append(float(parts[2]))
            except ValueError:
                pass
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}
        if watts:
            out["power_w"] = statistics.median(watts)  # median board power while timing
        return out


def oracle_block_sampler():
    """One branch-block of the 1024^2 workload (4608 tokens, hidden 3072) in the float64 oracle, as
    it stands: returns a function that runs it once and returns the seconds it took."""
    from oracle import moss_oracle as o
    from synth import ModelShape, make_residual, make_weights, numpy_weights

    shape = ModelShape(layers=1, hidden=3072, heads=24, ffn=8192)
    wn = numpy_weights(make_weights(shape, 7))
    x = make_residual(1, 4096 + N_TXT, 3072, 8)[0].double().numpy()
    ang = o.rope_angles(o.token_positions(64, 64, N_TXT))
    c = o.conditioning(0.5, wn)
    mod = o.block_modulation(c, wn["mod_w"][0], wn["mod_b"][0])
    lw = o.layer_weights(wn, 0)

    def run_once():
        t0 = time.perf_counter()
        o.block_forward(x, lw, mod, ang, shape.heads)
        return time.perf_counter() - t0

    return run_once


def _oracle_threads():
    from threadpoolctl import threadpool_info
    return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])


def cpu_baseline(run_once=None):
    """The oracle on one branch-block of the 1024^2 workload, timed once: forwards/s =
    1 / (42 * block time)."""
    run_once = run_once or oracle_block_sampler()
    dt = run_once()
    return {"value": 1.0 / (42 * dt), "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"one branch-block (4608 tokens x 3072, float64) timed once: {dt:.2f} s; "
                      f"forwards/s = 1/(42 x block time)"}


REFERENCE_SAMPLE = ("one branch-block of the 1024^2 workload per timed step (4608 tokens x hidden 3072, "
                    "float64 oracle), extrapolated to the step's 83 branch-blocks")


def run_reference(args):
    """The oracle as it stands, on the host cores: each of the --steps timed steps runs one
    branch-block of the workload (a bounded sample of the step's 83), and the step time is
    extrapolated from the mean block time.  Rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps = max(1, args.steps)
    warm = min(args.warmup, 1)
    run_once = oracle_block_sampler()
    for _ in range(warm):
        run_once()
    samples = [cpu_baseline(run_once) for _ in range(steps)]
    value = statistics.mean(s["value"] for s in samples)
    cb = dict(samples[-1], value=value, sample=REFERENCE_SAMPLE)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": 2000.0 / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": 4096 + N_TXT, "parallelism": "none"},
            "extrapolated": True, "timed_per_step": "one branch-block (4608 tokens x 3072)",
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_op(args):
    """Kernel-level timing on the 1024^2 shapes (batch 2, 4096 image + 512 text tokens):
    `block` runs one full-width block (hidden 3072, 24x128 heads, FFN 8192) in place,
    `attention` the attention kernel alone.  Prints one JSON line of per-class device time.
    Used for ncu captures of single kernels on a small, one-layer case."""
    import torch

    import diffusion_transformer_text_block_b200 as moss
    from synth import ModelShape, make_residual, make_weights

    shape = ModelShape(layers=1, hidden=3072, heads=24, ffn=8192)
    N = 4096 + N_TXT
    if args.op == "attention":
        g = torch.Generator(device="cuda").manual_seed(5)
        qkv = torch.randn(2, N, 3 * 3072, generator=g, device="cuda").to(torch.bfloat16)
        for _ in range(args.warmup):
            moss.op_attention(qkv, 24)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            moss.op_attention(qkv, 24)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        tf = 2 * flops_per_branch_layer(N)["attention"] / (ms / 1e3) / 1e12
        print(json.dumps({"op": "attention", "ms": round(ms, 4), "tflops": round(tf, 1)}), flush=True)
        return 0
    w = {k: v for k, v in make_weights(shape, 3, device="cuda").items()}
    model = moss.Model(shape, w, max_tokens=N, max_batch=2, max_latent_hw=128 * 128, max_steps=1)
    x = make_residual(2, N, 3072, 4, device="cuda")
    for _ in range(args.warmup):
        model.block_forward(0, x, 64, 64, N_TXT, 0.5)
    torch.cuda.synchronize()
    model.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        model.block_forward(0, x, 64, 64, N_TXT, 0.5)
    e1.record()
    torch.cuda.synchronize()
    prof = model.profile_read()
    fl = flops_per_branch_layer(N)
    out = {"op": "block", "ms_per_block": round(e0.elapsed_time(e1) / args.steps, 4)}
    for k, (n, tms) in prof.items():
        if n:
            out[k] = {"ms": round(tms / n, 4)}
            if k in fl:
                out[k]["tflops"] = round(2 * fl[k] / (tms / n / 1e3) / 1e12, 1)
    out["device_status"] = moss.device_status(clear=True)
    model.close()
    print(json.dumps(out), flush=True)
    return 0


def run_cfg_euler(args):
    """The standalone CFG + Euler kernel (moss_cfg_euler_step) on the 1024^2 and 2048^2 latents
    (128x128x32 and 256x256x32 FP32): x, v_c and v_u only.  Each launch takes the next of enough
    buffer sets that together exceed L2 twice over, so every launch streams from HBM.  Prints one JSON
    line: per size the mean device time per launch and the algorithmic HBM bytes (read x, v_c, v_u;
    write x: 16 B per element) over that time.  The launches are captured once in a CUDA graph and
    the graph is replayed between CUDA events, so the host's per-call cost (about 12 us through the
    Python binding, longer than the kernel itself) does not pace the device."""
    import torch

    import diffusion_transformer_text_block_b200 as moss

    peaks = read_peaks()
    out = {"op": "cfg_euler", "l2": "buffer sets rotated, 2 x L2 in total", "sizes": {}}
    for side in (1024, 2048):
        n = (side // 8) * (side // 8) * 32
        sets = max(2, int(2 * 126e6 // (12 * n)) + 1)
        bufs = [[torch.randn(n, device="cuda") for _ in range(3)] for _ in range(sets)]
        for i in range(max(args.warmup, 3)):
            x, c, u = bufs[i % sets]
            moss.cfg_euler_step(x, c, u, 3.0, 0.9, 0.8)
        torch.cuda.synchronize()
        launches = max(args.steps, 2 * sets)
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        with torch.cuda.stream(cap):
            with torch.cuda.graph(graph, stream=cap):
                for i in range(launches):
                    x, c, u = bufs[i % sets]
                    moss.cfg_euler_step(x, c, u, 3.0, 0.9, 0.8)
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / launches
        del graph
        gbs = 16.0 * n / (us * 1e-6) / 1e9
        out["sizes"][f"{side}^2"] = {"elements": n, "bytes_per_launch": 16 * n, "us_per_launch": round(us, 3),
                                     "gbs": round(gbs, 1), "hbm_frac": round(gbs / peaks["hbm_gbs"], 4),
                                     "launches": launches, "buffer_sets": sets}
        del bufs
    out["peak_source"] = f"{peaks['source']} hbm {peaks['hbm_gbs']} GB/s"
    out["device_status"] = moss.device_status(clear=True)
    print(json.dumps(out), flush=True)
    return 0


def run_c5(args):
    """The long-sequence stress workload: 2048^2 (16384 image tokens) with a 4096-token prompt
    (20480 tokens per branch), full 42-block DiT, CFG batch 2, skip layer 22, 10 Euler steps at
    shift 5.  Times --steps of those steps (default all 10) after --warmup, with per-class device
    time; prints one JSON line."""
    import torch

    import diffusion_transformer_text_block_b200 as moss
    from synth import FULL, make_text, make_weights

    H = W = 2048
    n_txt, n_steps = 4096, 10
    N = (H // 16) * (W // 16) + n_txt
    w = make_weights(FULL, 2, device="cuda")
    model = moss.Model(FULL, w, max_tokens=N, max_batch=2, max_latent_hw=(H // 8) * (W // 8), max_steps=1)
    tc = make_text(1, n_txt, FULL.hidden, 100, device="cuda")[0].contiguous()
    tu = make_text(1, n_txt, FULL.hidden, 200, device="cuda")[0].contiguous()
    x = torch.empty(H // 8, W // 8, 32, device="cuda")
    moss.init_noise(x, 42)
    steps = min(args.steps, n_steps)

    def step(i):
        model.denoise_step(x, tc, tu, H, W, i, n_steps, CFG, SHIFT, SKIP, *SLG)

    for i in range(min(args.warmup, 1)):
        step(i)
    torch.cuda.synchronize()
    model.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    prof = model.profile_read()
    peaks = read_peaks()
    bl = sum(2 * FULL.layers - (len(SKIP) if _slg_on(i, n_steps, *SLG) else 0) for i in range(steps))
    fl = flops_per_branch_layer(N)
    out = {"op": "c5", "workload": "2048^2, 16384 image + 4096 text tokens per branch, CFG batch 2, skip layer 22, "
           "10 Euler steps, shift 5, random-init 42-block DiT", "s_per_step": round(ms / 1e3, 4),
           "s_per_10_steps": round(ms * n_steps / 1e3, 3), "steps_timed": steps, "kernels": {}}
    total = 0.0
    for k, (n, tms) in prof.items():
        if not n:
            continue
        rec = {"launches": n, "ms": round(tms, 3)}
        total += tms
        if k in fl:
            tf = bl * fl[k] / (tms / 1e3) / 1e12
            rec["tflops"] = round(tf, 1)
            rec["frac"] = round(tf / peaks["bf16_tflops_sustained"], 4)
        out["kernels"][k] = rec
    for k in out["kernels"]:
        out["kernels"][k]["share"] = round(out["kernels"][k]["ms"] / total, 4)
    out["device_status"] = moss.device_status(clear=True)
    model.close()
    print(json.dumps(out), flush=True)
    return 0


def run_text(args):
    """The text path once per prompt: projection 4096 -> 3072 and two text-only blocks at full
    width, for the benchmark's 512-token prompt and the pages' 4096-token maximum.  Prints one JSON
    line: ms per call (CUDA events) and TFLOP/s of the algorithmic work."""
    import torch

    import diffusion_transformer_text_block_b200 as moss
    from synth import ModelShape, make_encoder_states, make_text_weights, make_weights

    shape = ModelShape(layers=1, hidden=3072, heads=24, ffn=8192)
    D, F = shape.hidden, shape.ffn
    w = {k: v for k, v in make_weights(shape, 3, device="cuda").items()}
    model = moss.Model(shape, w, max_tokens=4096, max_batch=1, max_latent_hw=64, max_steps=1)
    model.set_text_weights(make_text_weights(shape, 4, device="cuda"))
    out = {"op": "text"}
    for n in (N_TXT, 4096):
        enc = make_encoder_states(n, 5, device="cuda")
        res = torch.empty(n, D, device="cuda")
        for _ in range(args.warmup):
            model.text_refine(enc, out=res)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            model.text_refine(enc, out=res)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        flop = 2.0 * n * 4096 * D + 2 * (2.0 * n * D * (4 * D + 3 * F) + 4.0 * n * n * D)
        out[f"n{n}"] = {"ms": round(ms, 4), "tflops": round(flop / (ms / 1e3) / 1e12, 1)}
    out["device_status"] = moss.device_status(clear=True)
    model.close()
    print(json.dumps(out), flush=True)
    return 0


def run_accel(args):
    """Whole 1024^2 images (50 steps, CFG 3, shift 5, uncond skips layer 22 in slg [0.01, 1.0])
    through moss_sample and moss_sample_ex with the lossy accelerators (CFG truncation, the
    first-block step cache at the pages' default thresholds 0.02 and 0.03) and with three-pass
    skip-layer guidance (a third branch inside the window).  Random-init
    weights: how often the cache engages depends on the weights, so the reuse counts here say
    nothing about a trained model.  Prints one JSON line: seconds per image (CUDA events around
    each call) and the number of reused steps."""
    import torch

    import diffusion_transformer_text_block_b200 as moss
    from synth import FULL, make_text, make_weights

    w = make_weights(FULL, 2, device="cuda")
    model = moss.Model(FULL, w, max_tokens=4096 + N_TXT, max_batch=3, max_latent_hw=128 * 128, max_steps=50)
    tc = make_text(1, N_TXT, FULL.hidden, 100, device="cuda")[0].contiguous()
    tu = make_text(1, N_TXT, FULL.hidden, 200, device="cuda")[0].contiguous()
    kw = dict(steps=STEPS_PER_IMAGE, cfg=CFG, shift=SHIFT, seed=42, uncond_skip_layers=SKIP, slg_start=SLG[0],
              slg_stop=SLG[1])
    runs = [("plain", None), ("cfg_truncation_0.5", dict(cfg_truncation=0.5)),
            ("step_cache_0.02", dict(step_cache_threshold=0.02)), ("step_cache_0.03", dict(step_cache_threshold=0.03)),
            ("both_0.5_0.03", dict(cfg_truncation=0.5, step_cache_threshold=0.03)),
            ("three_pass_slg_2.0", dict(slg_scale=2.0))]
    model.sample(tc, tu, HEIGHT, WIDTH, **dict(kw, steps=2))  # warm-up
    torch.cuda.synchronize()
    out = {"op": "accel", "workload": "1024^2 image, 50 steps, CFG 3, random-init 42-block DiT", "runs": {}}
    base = None
    for name, opt in runs:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if opt is None:
            model.sample(tc, tu, HEIGHT, WIDTH, **kw)
            cached, change = [False] * STEPS_PER_IMAGE, []
        else:
            _, cached, change = model.sample_accelerated(tc, tu, HEIGHT, WIDTH, **kw, **opt)
        e1.record()
        torch.cuda.synchronize()
        s_img = e0.elapsed_time(e1) / 1e3
        base = base or s_img
        rec = {"s_per_image": round(s_img, 3), "speedup": round(base / s_img, 3), "reused_steps": int(sum(cached))}
        finite = [c for c in change if c == c]
        if finite:
            rec["change_min_max"] = [round(min(finite), 5), round(max(finite), 5)]
        out["runs"][name] = rec
    out["device_status"] = moss.device_status(clear=True)
    model.close()
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=STEPS_PER_IMAGE)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", choices=["block", "attention", "accel", "text", "c5", "cfg_euler"], default=None,
                    help="time one kernel class on the 1024^2 shapes instead of the denoising step; "
                         "'accel' times whole 50-step images with the lossy accelerators")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "accel":
        return run_accel(args)
    if args.op == "text":
        return run_text(args)
    if args.op == "c5":
        return run_c5(args)
    if args.op == "cfg_euler":
        return run_cfg_euler(args)
    if args.op:
        return run_op(args)

    import torch
    import torch.distributed as dist

    import diffusion_transformer_text_block_b200 as moss
    from synth import FULL, make_text, make_weights

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    w = make_weights(FULL, 2, device="cuda")
    model = moss.Model(FULL, w, max_tokens=4096 + N_TXT, max_batch=2, max_latent_hw=128 * 128, max_steps=50)
    tc = make_text(1, N_TXT, FULL.hidden, 100 + rank, device="cuda")[0].contiguous()
    tu = make_text(1, N_TXT, FULL.hidden, 200 + rank, device="cuda")[0].contiguous()
    x = torch.empty(HEIGHT // 8, WIDTH // 8, 32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i):
        model.denoise_step(x, tc, tu, HEIGHT, WIDTH, i % STEPS_PER_IMAGE, STEPS_PER_IMAGE, CFG, SHIFT, SKIP, *SLG)

    moss.init_noise(x, 42 + rank)
    for i in range(args.warmup):
        step(i)
    moss.init_noise(x, 42 + rank)
    # The warm-up left the schedule's modulation in the model; drop it, so that the first timed
    # step computes it for the whole schedule as moss_sample does once per image.
    model.modulation(0.5)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # The timed region times the launches of the two largest kernel classes (the dominant one is
    # the roofline's kernel); every timed launch adds two event records to the stream, so the
    # other classes are timed in a separate pass after it.
    timed_classes = ("gemm_gateup", "attention")
    model.profile_enable_classes(timed_classes)
    launches0 = moss.launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for i in range(args.steps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = moss.launch_count() - launches0
    ms = ev0.elapsed_time(ev1)
    prof_timed = model.profile_read()
    model.profile_enable(False)
    status = moss.device_status(clear=True)
    # per-class breakdown: a profiled pass over the same steps of the schedule (all classes)
    prof_steps = min(args.steps, 10)
    model.profile_enable(True)
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for i in range(prof_steps):
        step(i)
    p1.record(stream)
    torch.cuda.synchronize()
    prof = model.profile_read()
    prof_ms = p0.elapsed_time(p1)
    model.profile_enable(False)
    status = max(status, moss.device_status(clear=True))
    ms = max_over_ranks(ms, dist if world > 1 else None, "cuda")
    if world > 1:
        dist.barrier()
    value, ms_per_step = job_throughput(args.steps, world, ms)

    # roofline of the dominant kernel class (largest summed device time)
    N = 4096 + N_TXT
    fl = flops_per_branch_layer(N)
    bl = sum(step_branch_layers(i) for i in range(args.steps))
    peaks = read_peaks()
    # HBM-bound classes: algorithmic bytes over the timed steps.  LN-modulate reads an FP32 row
    # and writes a BF16 row (2 calls per branch-layer, N rows each, plus the final layer's image
    # rows per branch); CFG + Euler reads x, v_c, v_u and writes x (16 B per latent element).
    D = 3072
    bl_p = sum(step_branch_layers(i) for i in range(prof_steps))
    hbm_bytes = {
        "ln_mod": (2 * bl_p * N + 2 * 4096 * prof_steps) * D * 6.0,
        "cfg_euler": 16.0 * (HEIGHT // 8) * (WIDTH // 8) * 32 * prof_steps,
    }
    kernels = {}
    for name, (n, tms) in prof.items():
        entry = {"launches": n, "ms": round(tms, 3), "share": round(tms / prof_ms, 4) if prof_ms else None}
        if name in fl and tms > 0:
            tf = fl[name] * bl_p / (tms / 1e3) / 1e12
            entry["tflops"] = round(tf, 1)
            entry["frac"] = round(tf / peaks["bf16_tflops_sustained"], 4)
        if name in hbm_bytes and tms > 0:
            gbs = hbm_bytes[name] / (tms / 1e3) / 1e9
            entry["gbs"] = round(gbs, 1)
            entry["hbm_frac"] = round(gbs / peaks["hbm_gbs"], 4)
        kernels[name] = entry
    dom = max((k for k in timed_classes if prof_timed[k][1] > 0), key=lambda k: prof_timed[k][1])
    n_dom, ms_dom = prof_timed[dom]
    achieved = fl[dom] * bl / (ms_dom / 1e3) / 1e12
    roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1),
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops_sustained"], 4), "traffic": kernel_traffic(dom),
                "peak_source": f"{peaks['source']} bf16 sustained",
                "flop_per_launch": fl[dom] * bl / max(n_dom, 1)}
    step_flops = sum(fl.values()) * bl / args.steps
    tc_frac = step_flops * args.steps / (ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"]

    # End to end through the C-ABI call with host buffers (moss_denoise_step_host): every step
    # copies the latent and both prompts from pinned host memory to the device, runs the step and
    # copies the latent back, all inside the call; the call returns with the result in host memory.
    e2e = None
    if args.e2e_steps > 0:
        hx = x.cpu().pin_memory()
        htc = tc.cpu().pin_memory()
        htu = tu.cpu().pin_memory()
        # Untimed warm-up of the host-buffer path: its first call allocates the staging buffers.
        hx0 = hx.clone()
        model.denoise_step_host(hx, htc, htu, HEIGHT, WIDTH, 0, STEPS_PER_IMAGE, CFG, SHIFT, SKIP, *SLG)
        hx.copy_(hx0)
        model.modulation(0.5)  # as above: the first e2e step computes the schedule's modulation
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(args.e2e_steps):
            model.denoise_step_host(hx, htc, htu, HEIGHT, WIDTH, i % STEPS_PER_IMAGE, STEPS_PER_IMAGE, CFG, SHIFT,
                                    SKIP, *SLG)
        a1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(a0.elapsed_time(a1), dist if world > 1 else None, "cuda")
        e2e = {"value": job_throughput(args.e2e_steps, world, ems)[0], "unit": UNIT,
               "h2d_bytes_per_step": hx.numel() * 4 + htc.numel() * 4 + htu.numel() * 4,
               "d2h_bytes_per_step": hx.numel() * 4, "steps": args.e2e_steps,
               "call": "moss_denoise_step_host (pinned host buffers, copies and a stream wait inside the call)"}

    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    cb = None if args.no_cpu_baseline or world > 1 else cpu_baseline()
    s_per_image = ms_per_step / 1e3 * STEPS_PER_IMAGE
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world, "seq_len": N, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: 9.9 GB of weights stream through each step"},
        "s_per_step": round(ms_per_step / 1e3, 4),
        "s_per_image": round(s_per_image, 3),
        "s_per_image_note": "measured over the timed steps" if args.steps == STEPS_PER_IMAGE else
                            "50 x mean s/step of the timed steps",
        "tc_frac_step": round(tc_frac, 4),
        "roofline": roofline, "kernels": kernels,
        "kernels_note": f"per-class device time from a profiled pass of {prof_steps} steps after the timed region "
                        "(the timed region itself times only the gemm_gateup and attention launches); the CFG + "
                        "Euler update runs inside the output projection (class 'other'), so 'cfg_euler' has no "
                        "launches in the step; bench.py --op cfg_euler times the standalone kernel",
        "cpu_baseline": cb, "e2e": e2e,
        "clocks": clocks.summary(), "gpu_launches": launches, "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
