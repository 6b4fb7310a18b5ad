#!/usr/bin/env python
"""Benchmark: one 50-block denoising step of the MiniMax-H3-Image DiT at a
4096^2 canvas (16,384 image tokens + 512 text tokens), through libh3dit.

    python bench.py [--gpus N --steps K --warmup W] [--head-dim 96|128]
    python bench.py --impl reference          # the CPU oracle on a bounded sample
    python bench.py --only attention          # one kernel kind alone (for profilers)
    python bench.py --oracle-configs          # the CPU oracle on every workload shape

Rank 0 prints one JSON line. Besides the contract's keys it carries the
per-step median/min/max, the same step replayed from a CUDA graph, the 6-step
total, the GEMM and attention TFLOP/s, ms per block at the other workload
shapes (small block, 2048^2, 4096^2, the edit request with four references)
and the MXFP8 variant of the step. Multi-GPU runs are independent replicas (the
step does not shard): every rank runs its own step on its own weights, the
timed region is bracketed by barriers and the slowest rank's time is used.
Weights are random-init bf16 (44 GB for 50 blocks at head_dim 96), generated
on the device from a seed; all inputs are larger than L2, so no flush is
needed between steps.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

D, H, F, L = 5376, 56, 14336, 50
N_TXT, GRID = 512, 128
N_TOK = N_TXT + GRID * GRID
METRIC = "ms per 50-block 4096^2 denoise step"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet dense tensor peaks (no 2:4 sparsity), for the fractions
# reported beside the measured-peak ones.
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_FP8_TFLOPS = 4500.0
C_LAT = 24  # latent channels (16x VAE, 24 channels; 2x2 patches of 96 features)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="h3dit", choices=["h3dit", "reference"])
    ap.add_argument("--head-dim", type=int, default=96, choices=[96, 128])
    ap.add_argument("--only", default=None,
                    choices=["attention", "qkv", "out_proj", "ffn1", "ffn2", "rmsnorm", "adaln",
                             "vae"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-mxfp8", action="store_true")
    ap.add_argument("--no-vae", action="store_true",
                    help="skip the VAE decoder timing")
    ap.add_argument("--no-sp", action="store_true",
                    help="skip the one-GPU timing of a block under Ulysses SP4 (fused exchanges)")
    ap.add_argument("--no-streaming", action="store_true",
                    help="skip the layerwise weight-streaming timings")
    ap.add_argument("--no-denoise", action="store_true",
                    help="skip the 6-step sampling loop timing (h3dit_denoise)")
    ap.add_argument("--no-graph", action="store_true", help="skip the graph-replayed step timing")
    ap.add_argument("--oracle-configs", action="store_true",
                    help="time the CPU oracle on every workload shape (minutes) and exit")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-block timings of the other workload shapes")
    ap.add_argument("--mx", action="store_true",
                    help="with --only qkv/out_proj/ffn1/ffn2: the MXFP8 linear")
    return ap.parse_args()


def workload_name(dh: int) -> str:
    return (f"50-block DiT denoise step, 4096^2 canvas: {GRID}x{GRID} image + {N_TXT} text "
            f"tokens (joint {N_TOK}), hidden {D}, {H} heads x {dh}, GELU FFN {F}, bf16")


def flops_per_launch(kind: str, n: int, dh: int) -> float:
    I = H * dh
    return {"qkv": 2.0 * n * D * 3 * I, "attention": 4.0 * n * n * I,
            "out_proj": 2.0 * n * I * D, "ffn1": 2.0 * n * D * F,
            "ffn2": 2.0 * n * F * D}.get(kind, 0.0)


def bytes_per_launch(kind: str, n: int, dh: int, blocks: int = L) -> float:
    """Algorithmic HBM bytes of the memory-bound kernels."""
    return {"rmsnorm": n * D * (4 + 2) + 2 * D * 4,
            "adaln": blocks * 6 * D * (D * 2 + 4 + 4) + D * 4,
            "time_embed": (D * 256 + D * D + 3 * D) * 4,
            "pack": n * D * (2 + 4), "rope_table": n * (dh // 2) * 8}.get(kind, 0.0)


def step_flops(n: int, dh: int) -> float:
    I = H * dh
    return L * (8.0 * n * D * I + 4.0 * n * D * F + 4.0 * n * n * I)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return FALLBACK_PEAKS, "fallback"


def traffic_for(kind: str, dh: int):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel's sources as they are now (every listed file's sha256 must
    match); else None."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kind}_dh{dh}.txt")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as fh:
        for line in fh:
            if ":" in line:
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    srcs = fields.get("sources", "").split()
    shas = fields.get("sha256", "").split()
    if not srcs or len(srcs) != len(shas) or "dram_bytes_per_launch" not in fields:
        return None
    for src, sha in zip(srcs, shas):
        with open(os.path.join(ROOT, src), "rb") as fh:
            if hashlib.sha256(fh.read()).hexdigest() != sha:
                return None
    return float(fields["dram_bytes_per_launch"])


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- device setup

def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def slowest_rank(value: float, dist, device="cuda") -> float:
    """The largest of every rank's value (the job is as slow as its slowest
    replica); identity without a process group."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def time_steps(ctx, steps, warmup, x_img, x_txt, grids, barrier, dist):
    """W warm-up steps, then K steps between barriers; (ms per step, profile,
    launches), the time being the slowest rank's."""
    import torch

    ts = timesteps(warmup + steps)
    for i in range(warmup):
        ctx.step(ts[i], x_img, grids, x_txt)
    barrier()
    if ctx.sync_status() != 0:
        raise RuntimeError("warm-up failed")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ctx.profile_begin()
    n0 = ctx.launch_count()
    e0.record(stream)
    for i in range(steps):
        ctx.step(ts[warmup + i], x_img, grids, x_txt)
    e1.record(stream)
    barrier()
    launches = ctx.launch_count() - n0
    prof = ctx.profile_end()
    elapsed = slowest_rank(e0.elapsed_time(e1), dist)
    if ctx.sync_status() != 0:
        raise RuntimeError("timed steps failed")
    return elapsed / steps, prof, launches


def make_model(dh: int, seed: int):
    import torch

    from image_generation_b200 import h3dit as Hb

    I = H * dh
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)

    def w(*shape, dtype=torch.bfloat16):
        return (torch.randn(*shape, device="cuda", generator=g) * 0.02).to(dtype)

    tw = {"w_t1": w(D, 256, dtype=torch.float32), "b_t1": torch.zeros(D, device="cuda"),
          "w_t2": w(D, D, dtype=torch.float32), "b_t2": torch.zeros(D, device="cuda")}
    blocks = [{"w_qkv": w(3 * I, D), "w_o": w(D, I), "w_ff1": w(F, D), "w_ff2": w(D, F),
               "w_ada": w(6 * D, D), "b_ada": torch.zeros(6 * D, device="cuda")}
              for _ in range(L)]
    cfg = Hb.make_config(D, H, dh, F, L, N_TOK)
    return Hb.Context(cfg, tw, blocks), tw, blocks


def tokens(seed: int):
    import torch

    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x_txt = torch.randn(N_TXT, D, device="cuda", generator=g).bfloat16()
    x_img = torch.randn(GRID * GRID, D, device="cuda", generator=g).bfloat16()
    return x_txt, x_img


def timesteps(k: int):
    return [1.0 - (i % 6) / 6.0 for i in range(k)]


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(dh: int, rows_a: int = 32, rows_b: int | None = 544, seed: int = 0):
    """Time the oracle on one block of the 4096^2 step for two query-row
    samples (keys and values always over all tokens) and extrapolate linearly
    to all rows and to the 50 blocks of a step, plus the per-step timestep MLP
    and AdaLN projections: an estimate, not a timed step. Returns (ms per step,
    description, threads, CPU seconds). With rows_b None only the first sample
    runs (a warm-up) and the estimate is None."""
    import numpy as np

    from image_generation_b200 import synth
    from oracle import dit_block as O

    dims = synth.Dims(D, H, dh, F)
    cfg = O.config_for(D, H, dh, F)
    w = synth.block_weights(dims, seed)
    tw = synth.time_weights(dims, seed)
    pos = O.token_positions(N_TXT, [(0, GRID, GRID)])
    x = synth.tokens(N_TOK, D, seed, "x").astype(np.float64)
    rng = np.random.default_rng(seed)
    t0 = time.perf_counter()
    c = O.timestep_condition(0.5, tw, cfg)
    t_time = time.perf_counter() - t0
    t0 = time.perf_counter()
    mod = O.adaln_modulation(c, w["w_ada"], w["b_ada"])
    t_ada = time.perf_counter() - t0
    times = []
    for r in (rows_a, rows_b):
        if r is None:
            return None, "", _blas_threads(), times[0]
        rows = np.sort(rng.choice(N_TOK, r, replace=False))
        t0 = time.perf_counter()
        O.block_forward(x, mod, w, pos, cfg, rows=rows)
        times.append(time.perf_counter() - t0)
    slope = max((times[1] - times[0]) / (rows_b - rows_a), 0.0)
    fixed = max(times[0] - slope * rows_a, 0.0)
    block_s = fixed + slope * N_TOK
    step_ms = 1e3 * (t_time + L * t_ada + L * block_s)
    threads = _blas_threads()
    desc = (f"estimate: oracle (float64 numpy) on one block of the step for {rows_a} and {rows_b} "
            f"query rows (K/V over all {N_TOK} tokens): {times[0]:.2f} s and {times[1]:.2f} s; "
            f"extrapolated linearly to {N_TOK} rows and x{L} blocks, plus the timestep MLP "
            f"({t_time * 1e3:.1f} ms) and {L} AdaLN projections ({t_ada * 1e3:.1f} ms each)")
    return step_ms, desc, threads, sum(times) + t_time + t_ada


def oracle_block_2k(dh: int, seed: int = 0):
    """The oracle timed on one whole block of the 2048^2 workload (4608
    tokens, every row): a measured CPU figure, not an extrapolation. Returns
    (ms, description, threads)."""
    import numpy as np

    from image_generation_b200 import synth
    from oracle import dit_block as O

    w = synth.WORKLOADS["block_2k" if dh == 96 else "block_2k_dh128"]
    d = w.dims
    cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
    bw = synth.block_weights(d, seed)
    tw = synth.time_weights(d, seed)
    inp = synth.workload_inputs(w)
    x = O.pack(inp["x_txt"], inp["x_img"])
    pos = O.token_positions(w.n_txt, w.grids)
    t0 = time.perf_counter()
    mod = O.adaln_modulation(O.timestep_condition(inp["t"], tw, cfg), bw["w_ada"], bw["b_ada"])
    O.block_forward(x, mod, bw, pos, cfg)
    ms = 1e3 * (time.perf_counter() - t0)
    return ms, (f"oracle (float64 numpy), one whole 2048^2 block ({w.n_tokens} tokens, "
                f"head_dim {d.head_dim}) with its timestep MLP and AdaLN projection, timed"), \
        _blas_threads()


def run_oracle_configs(args):
    """The oracle (float64 numpy) timed on this host: the small block and the
    2048^2 block in full, the 4096^2 block and the edit request by sampled
    query rows extrapolated linearly (labelled), and the 50-block step from
    the 4096^2 block; plus the C oracle's plain-fp32 build on the small block.
    One JSON line; test infrastructure, not a bench value."""
    import numpy as np

    from image_generation_b200 import synth
    from oracle import dit_block as O

    dh = args.head_dim
    out = {}
    for name in ("small_block", "block_2k", "block_4k", "edit_4ref"):
        w = synth.WORKLOADS[name if dh == 96 or name == "small_block" else name + "_dh128"]
        d = w.dims
        cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
        bw = synth.block_weights(d, w.seed)
        tw = synth.time_weights(d, w.seed)
        inp = synth.workload_inputs(w)
        x = O.pack(inp["x_txt"], inp["x_img"])
        pos = O.token_positions(w.n_txt, w.grids)
        mod = O.adaln_modulation(O.timestep_condition(inp["t"], tw, cfg), bw["w_ada"], bw["b_ada"])
        if w.n_tokens <= 5000:
            t0 = time.perf_counter()
            O.block_forward(x, mod, bw, pos, cfg)
            out[name] = {"s_per_block": round(time.perf_counter() - t0, 2), "tokens": w.n_tokens,
                         "how": "full block"}
        else:
            rng = np.random.default_rng(0)
            O.block_forward(x, mod, bw, pos, cfg, rows=np.arange(8))  # untimed: first-touch costs
            t = []
            for r in (32, 544):
                rows = np.sort(rng.choice(w.n_tokens, r, replace=False))
                t0 = time.perf_counter()
                O.block_forward(x, mod, bw, pos, cfg, rows=rows)
                t.append(time.perf_counter() - t0)
            slope = max((t[1] - t[0]) / 512, 0.0)
            est = max(t[0] - 32 * slope, 0.0) + slope * w.n_tokens
            out[name] = {"s_per_block": round(est, 1), "tokens": w.n_tokens,
                         "how": f"extrapolated from 32 and 544 query rows ({t[0]:.1f} s, {t[1]:.1f} s)"}
    blk = out["block_4k"]["s_per_block"]
    out["step_4k"] = {"s_per_step": round(L * blk, 0), "how": f"extrapolated: {L} x the 4096^2 block"}
    out["six_steps_4k"] = {"s": round(6 * L * blk, 0), "how": "extrapolated: 6 steps"}
    # the independent C oracle, plain fp32 loops on one core, on the small block
    try:
        from oracle import ref_c

        ref = ref_c.load("f32")
        w = synth.WORKLOADS["small_block"]
        d = w.dims
        cfg = O.config_for(d.hidden, d.heads, d.head_dim, d.ffn)
        bw = synth.block_weights(d, w.seed)
        inp = synth.workload_inputs(w)
        x = O.pack(inp["x_txt"], inp["x_img"])
        mod = O.adaln_modulation(O.timestep_condition(inp["t"], synth.time_weights(d, w.seed), cfg),
                                 bw["w_ada"], bw["b_ada"])
        pos = O.token_positions(w.n_txt, w.grids)
        t0 = time.perf_counter()
        ref.block_forward(x, mod, bw, pos, heads=d.heads, head_dim=d.head_dim,
                          sections=cfg.rope_sections)
        out["small_block_c_f32"] = {"s_per_block": round(time.perf_counter() - t0, 2),
                                    "tokens": w.n_tokens, "how": "C oracle, fp32, 1 core"}
    except (OSError, RuntimeError) as e:  # no C compiler on this host
        out["small_block_c_f32"] = {"unavailable": str(e).splitlines()[0]}
    print(json.dumps({"oracle_timing": out, "head_dim": dh, "cores": _blas_threads(),
                      "dtype": "f64"}), flush=True)
    return 0


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------- arms

def run_reference(args):
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    vals = []
    desc, threads = "", 1
    for _ in range(args.warmup):  # untimed: one short sample each
        oracle_sample(args.head_dim, rows_a=8, rows_b=None)
    t_all = time.perf_counter()
    for _ in range(args.steps):
        v, desc, threads, _ = oracle_sample(args.head_dim)
        vals.append(v)
    wall = time.perf_counter() - t_all
    value = sum(vals) / len(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "ms",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(value, 1), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, random-init weights)",
        "config": {"workload": workload_name(args.head_dim), "n_blocks": L, "tokens": N_TOK,
                   "head_dim": args.head_dim, "global_batch": world,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (~44 GB of weights read per step)"},
        "cpu_baseline": {"value": round(value, 1), "unit": "ms", "cores": threads,
                         "kind": "oracle", "estimated": True, "sample": desc},
        "e2e": {"value": round(value, 1), "unit": "ms", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 1),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_only(args):
    """One kernel kind alone at the step's shape (for ncu captures); "vae" is
    the VAE decoder on the 4096^2 canvas's latent, --warmup + --steps decodes."""
    import torch

    from image_generation_b200 import h3dit as Hb

    if args.only == "vae":
        out = vae_timing(reps=max(args.steps, 1), warmup=args.warmup, graph=False)
        print(json.dumps({"kernel": "vae_decode", **out}), flush=True)
        return 0

    dh = args.head_dim
    I = H * dh
    torch.manual_seed(0)
    mx = bool(args.mx) and args.only in ("qkv", "out_proj", "ffn1", "ffn2")
    cfg = Hb.make_config(D, H, dh, F, 1, N_TOK,
                         precision=Hb.H3DIT_PRECISION_MXFP8 if mx else Hb.H3DIT_PRECISION_BF16)
    g = lambda *s: (torch.randn(*s, device="cuda") * 0.02).bfloat16()
    tw = {"w_t1": torch.randn(D, 256, device="cuda") * 0.02, "b_t1": torch.zeros(D, device="cuda"),
          "w_t2": torch.randn(D, D, device="cuda") * 0.02, "b_t2": torch.zeros(D, device="cuda")}
    need = {"qkv": "w_qkv", "out_proj": "w_o", "ffn1": "w_ff1", "ffn2": "w_ff2"}.get(args.only)
    shapes = {"w_qkv": (3 * I, D), "w_o": (D, I), "w_ff1": (F, D), "w_ff2": (D, F), "w_ada": (6 * D, D)}
    # an MXFP8 context quantizes all four linears at create: they must be full size
    blk = {k: (g(*shp) if k in (need, "w_ada") or mx else torch.zeros(8, device="cuda").bfloat16())
           for k, shp in shapes.items()}
    blk["b_ada"] = torch.zeros(6 * D, device="cuda")
    ctx = Hb.Context(cfg, tw, [blk])
    n = N_TOK
    if args.only == "attention":
        qkv = torch.randn(n, 3 * I, device="cuda").bfloat16()
        o = torch.empty(n, I, device="cuda", dtype=torch.bfloat16)
        fn = lambda: ctx.attention(qkv[:, :I], qkv[:, I:2 * I], qkv[:, 2 * I:], 3 * I, o, I, n)
    elif mx:
        # the block's own MXFP8 linear (weights quantized at create), through
        # the kernel the MXFP8 step runs for it
        w = blk[need]
        a = torch.randn(n, w.shape[1], device="cuda").bfloat16()
        aq = torch.empty(n, w.shape[1], dtype=torch.uint8, device="cuda")
        asf = torch.empty(Hb.mx_scale_bytes(n, w.shape[1]), dtype=torch.uint8, device="cuda")
        ctx.mx_quantize(a, aq, asf)
        which = {"qkv": Hb.H3DIT_LINEAR_QKV, "out_proj": Hb.H3DIT_LINEAR_OUT,
                 "ffn1": Hb.H3DIT_LINEAR_FFN1, "ffn2": Hb.H3DIT_LINEAR_FFN2}[args.only]
        if args.only == "qkv":
            table = torch.empty(n, dh // 2, 2, device="cuda")
            ctx.rope_table([(0, GRID, GRID)], N_TXT, table)
            out = torch.empty(n, w.shape[0], device="cuda", dtype=torch.bfloat16)
            fn = lambda: ctx.block_linear_mx(0, which, aq, asf, out, rope_table=table)
        elif args.only == "ffn1":
            out = torch.empty(n, w.shape[0], device="cuda", dtype=torch.uint8)
            osf = torch.empty(Hb.mx_scale_bytes(n, w.shape[0]), dtype=torch.uint8, device="cuda")
            fn = lambda: ctx.block_linear_mx(0, which, aq, asf, out, out_sf=osf)
        else:
            x = torch.randn(n, D, device="cuda")
            gate = torch.full((D,), 0.1, device="cuda")
            fn = lambda: ctx.block_linear_mx(0, which, aq, asf, x, gate=gate)
    elif args.only in ("qkv", "ffn1"):
        xm = torch.randn(n, D, device="cuda").bfloat16()
        table = torch.empty(n, dh // 2, 2, device="cuda")
        ctx.rope_table([(0, GRID, GRID)], N_TXT, table)
        out = torch.empty(n, blk[need].shape[0], device="cuda", dtype=torch.bfloat16)
        epi = Hb.H3DIT_EPI_QKV_ROPE if args.only == "qkv" else Hb.H3DIT_EPI_GELU
        fn = lambda: ctx.linear(epi, xm, blk[need], out, rope_table=table)
    elif args.only in ("out_proj", "ffn2"):
        a = torch.randn(n, blk[need].shape[1], device="cuda").bfloat16()
        x = torch.randn(n, D, device="cuda")
        gate = torch.full((D,), 0.1, device="cuda")
        fn = lambda: ctx.linear(Hb.H3DIT_EPI_GATED_RESIDUAL, a, blk[need], x, gate=gate)
    elif args.only == "rmsnorm":
        x = torch.randn(n, D, device="cuda")
        z = torch.zeros(D, device="cuda")
        out = torch.empty(n, D, device="cuda", dtype=torch.bfloat16)
        fn = lambda: ctx.rmsnorm_modulate(x, z, z, out)
    else:  # adaln, one block
        c = torch.randn(D, device="cuda")
        mod = torch.empty(1, 6, D, device="cuda")
        fn = lambda: ctx.adaln_project(c, 0, 1, mod)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ctx.profile_begin()
    for _ in range(args.steps):
        fn()
    prof = ctx.profile_end()
    assert ctx.sync_status() == 0
    ms, cnt = prof[args.only]
    per = ms / max(cnt, 1)
    fl = flops_per_launch(args.only, n, dh)
    by = bytes_per_launch(args.only, n, dh, blocks=1)
    out = {"kernel": args.only + ("_mxfp8" if args.mx else ""), "head_dim": dh, "tokens": n,
           "launches": cnt, "ms_per_launch": per}
    if fl:
        out["tflops"] = fl / per / 1e9
    if by:
        out["gbs"] = by / per / 1e6
    print(json.dumps(out), flush=True)
    return 0


def block_timings(dh: int) -> dict:
    """ms per block (block_forward, mod computed from t) at the other workload
    shapes: the small block (head_dim 96 only), the 2048^2 and 4096^2 canvases
    and the edit request with four references; random device weights, median
    of 5, with the attention and GEMM rates from the library's events."""
    import torch

    from image_generation_b200 import h3dit as Hb
    from image_generation_b200 import synth

    out = {}
    names = ["small_block", "block_2k", "block_4k", "edit_4ref"]
    if dh == 128:
        names = ["block_2k_dh128", "block_4k_dh128", "edit_4ref_dh128"]
    for name in names:
        w = synth.WORKLOADS[name]
        d = w.dims
        I = d.heads * d.head_dim
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        r = lambda *shape: (torch.randn(*shape, device="cuda", generator=g) * 0.02).bfloat16()
        tw = {"w_t1": torch.randn(d.hidden, 256, device="cuda", generator=g) * 0.02,
              "b_t1": torch.zeros(d.hidden, device="cuda"),
              "w_t2": torch.randn(d.hidden, d.hidden, device="cuda", generator=g) * 0.02,
              "b_t2": torch.zeros(d.hidden, device="cuda")}
        blk = {"w_qkv": r(3 * I, d.hidden), "w_o": r(d.hidden, I), "w_ff1": r(d.ffn, d.hidden),
               "w_ff2": r(d.hidden, d.ffn), "w_ada": r(6 * d.hidden, d.hidden),
               "b_ada": torch.zeros(6 * d.hidden, device="cuda")}
        ctx = Hb.Context(Hb.make_config(d.hidden, d.heads, d.head_dim, d.ffn, 1, w.n_tokens), tw, [blk])
        n_img = w.n_tokens - w.n_txt
        x_txt = torch.randn(w.n_txt, d.hidden, device="cuda", generator=g).bfloat16()
        x_img = torch.randn(n_img, d.hidden, device="cuda", generator=g).bfloat16()
        grids = list(w.grids)
        for _ in range(2):
            ctx.block_forward(0, 0.5, x_img, grids, x_txt)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        ctx.profile_begin()
        ev[0].record()
        for i in range(5):
            ctx.block_forward(0, 0.5, x_img, grids, x_txt)
            ev[i + 1].record()
        torch.cuda.synchronize()
        prof = ctx.profile_end()
        if ctx.sync_status() != 0:
            raise RuntimeError(f"block timing failed for {name}")
        ms = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(5))
        n = w.n_tokens
        att_ms, att_cnt = prof["attention"]
        gemm = ("qkv", "out_proj", "ffn1", "ffn2")
        g_ms = sum(prof[k][0] for k in gemm)
        g_fl = 5 * (8.0 * n * d.hidden * I + 4.0 * n * d.hidden * d.ffn)
        out[name] = {"ms": round(ms[2], 3), "tokens": n, "head_dim": d.head_dim,
                     "tflops": round(block_flops(n, d) / ms[2] / 1e9, 1),
                     "attention_tflops": round(4.0 * n * n * I * att_cnt / att_ms / 1e9, 1),
                     "gemm_tflops": round(g_fl / g_ms / 1e9, 1)}
        ctx.close()
        del blk, tw
    return out


def streamed_set(k: int, placement: str) -> set:
    """Which of the L blocks stream from the host when k stay resident:
    "tail" streams blocks k .. L-1; "spread" spaces the L - k streamed blocks
    evenly through the step, so that each one's copy overlaps the compute of
    the resident blocks around it as well as of the previous streamed block."""
    if placement == "tail":
        return set(range(k, L))
    m = L - k
    return {l for l in range(L) if (l + 1) * m // L - l * m // L == 1}


def streaming_timings(tw, blocks, x_txt, x_img, grids, dh,
                      residents=((24, "tail"), (24, "spread"), (8, "spread")), steps=2,
                      host_copies=4):
    """The 50-block 4096^2 step with only k blocks' weights on the device
    (placed as streamed_set says) and the rest streamed from pinned host
    memory through two staging slots (h3dit_attach_staging). The host blocks
    cycle through
    `host_copies` distinct pinned copies of the model's own blocks (the bytes
    moved per step are the same as with 50 - k distinct blocks; the step's
    output is not compared here - the tests check streamed steps bit for bit
    against resident ones). Returns {k: ms per step, ...} with the bytes
    crossing PCIe per step."""
    import torch

    from image_generation_b200 import h3dit as Hb

    host = [{k: v.cpu().pin_memory() for k, v in blocks[L - 1 - i].items()}
            for i in range(host_copies)]
    block_bytes = sum(v.numel() * v.element_size() for v in host[0].values())
    out = {}
    for k, placement in residents:
        streamed = streamed_set(k, placement)
        assert len(streamed) == L - k
        mixed = [host[l % host_copies] if l in streamed else blocks[l] for l in range(L)]
        ctx = Hb.Context(Hb.make_config(D, H, dh, F, L, N_TOK), tw, mixed)
        ctx.attach_staging()
        ts = timesteps(steps + 1)
        ctx.step(ts[0], x_img, grids, x_txt)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            ctx.step(ts[i + 1], x_img, grids, x_txt)
        e1.record()
        torch.cuda.synchronize()
        if ctx.sync_status() != 0:
            raise RuntimeError(f"streamed step failed (k={k})")
        ms = e0.elapsed_time(e1) / steps
        moved = (L - k) * block_bytes
        name = f"resident_{k}" if placement == "tail" else f"resident_{k}_{placement}"
        out[name] = {"ms_per_step": round(ms, 1), "streamed_blocks": L - k, "placement": placement,
                                "h2d_bytes_per_step": moved,
                                "h2d_gbs": round(moved / ms / 1e6, 1)}
        ctx.close()
    del host
    return out


def vae_flops(n_tok: int, tile: int, W=1280, M=5120, layers=24, C=24) -> float:
    """Algorithmic flops of a decode: the linears per token, plus 4 n^2 W per
    tile and layer for the attention over a tile's n tokens."""
    n = tile * tile
    lin = n_tok * (2 * C * W + layers * 2 * (4 * W * W + 2 * W * M) + 2 * W * 768)
    return float(lin + layers * (n_tok // n) * 4 * n * n * W)


def vae_timing(reps: int = 5, warmup: int = 2, graph: bool = True) -> dict:
    """The image VAE's 24-layer ViT decoder (width 1280, 10 heads x 128, MLP
    5120, 32 x 32 latent tiles) decoding the 4096^2 canvas's latent
    [24, 256, 256] (64 tiles, 65,536 tokens) on random device weights: ms per
    decode eagerly and replayed from a CUDA graph, TFLOP/s, kernel shares."""
    import torch

    from image_generation_b200 import h3dit as Hb

    W, M, L_, T = 1280, 5120, 24, 32
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    mat = lambda *s: (torch.randn(*s, device="cuda", generator=g) * 0.02).bfloat16()
    vec = lambda n, base=0.0: torch.randn(n, device="cuda", generator=g) * 0.02 + base
    layers = [{"ln1_g": vec(W, 1.0), "ln1_b": vec(W), "w_qkv": mat(3 * W, W), "b_qkv": vec(3 * W),
               "w_o": mat(W, W), "b_o": vec(W), "ln2_g": vec(W, 1.0), "ln2_b": vec(W),
               "w_1": mat(M, W), "b_1": vec(M), "w_2": mat(W, M), "b_2": vec(W)}
              for _ in range(L_)]
    weights = {"w_in": torch.randn(W, 24, device="cuda", generator=g) * 0.2, "b_in": vec(W),
               "layers": layers, "lnf_g": vec(W, 1.0), "lnf_b": vec(W), "w_out": mat(768, W),
               "b_out": vec(768)}
    hl = 2 * GRID  # latent side: 16x VAE downsampling of the 4096^2 canvas
    cfg = Hb.make_vae_config(W, 10, 128, M, L_, T, 24, hl * hl)
    dec = Hb.VaeDecoder(cfg, weights)
    z = torch.randn(24, hl, hl, device="cuda", generator=g)
    img = torch.empty(3, 16 * hl, 16 * hl, device="cuda")
    for _ in range(warmup):
        dec.decode(z, img)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dec.profile_begin()
    e0.record()
    for _ in range(reps):
        dec.decode(z, img)
    e1.record()
    torch.cuda.synchronize()
    prof = dec.profile_end()
    ms = e0.elapsed_time(e1) / reps
    g_ms = None
    if graph:
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg):
            dec.decode(z, img)
        cg.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            cg.replay()
        e1.record()
        torch.cuda.synchronize()
        g_ms = e0.elapsed_time(e1) / reps
        del cg
    if dec.sync_status() != 0 or not bool(torch.isfinite(img).all()):
        raise RuntimeError("VAE decode failed")
    fl = vae_flops(hl * hl, T)
    tot = sum(v[0] for v in prof.values()) or 1.0
    att_ms, att_n = prof["attention"]
    att_fl = L_ * (hl * hl // (T * T)) * 4.0 * (T * T) ** 2 * W
    out = {"ms": round(ms, 2), "graph_ms": None if g_ms is None else round(g_ms, 2),
           "tokens": hl * hl,
           "tiles": hl * hl // (T * T), "image": [3, 16 * hl, 16 * hl],
           "tflops": round(fl / ms / 1e9, 1),
           "attention_tflops": round(att_fl * reps / att_ms / 1e9, 1) if att_n else None,
           "kernel_share": {k: round(v[0] / tot, 4) for k, v in prof.items() if v[1]}}
    dec.close()
    return out


def denoise_timing(ctx, x_txt, rank, world, barrier, dist, stream, reps: int = 2) -> dict:
    """The whole 6-step sampling loop in one call (h3dit_denoise) on the 4096^2
    latent [24, 256, 256]: on the device, and end to end with the noise and
    the text states copied in from pinned host memory and the denoised latent
    copied back, all inside the timed region."""
    import torch

    g = torch.Generator(device="cuda")
    g.manual_seed(2000 + rank)
    k4 = 4 * C_LAT
    rnd = lambda *s: torch.randn(*s, device="cuda", generator=g) * 0.02
    io = {"w_in": rnd(D, k4), "b_in": torch.zeros(D, device="cuda"), "w_mod": rnd(2 * D, D),
          "b_mod": torch.zeros(2 * D, device="cuda"), "w_out": rnd(k4, D),
          "b_out": torch.zeros(k4, device="cuda")}
    shape = (C_LAT, 2 * GRID, 2 * GRID)
    noise = torch.randn(*shape, device="cuda", generator=g)
    lat = torch.empty_like(noise)
    h_noise = torch.empty(shape, pin_memory=True)
    h_noise.copy_(noise)
    h_txt = torch.empty(x_txt.shape, dtype=x_txt.dtype, pin_memory=True)
    h_txt.copy_(x_txt)
    h_out = torch.empty(shape, pin_memory=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lat.copy_(noise)
    ctx.denoise(io, lat, x_txt, 6)  # warm-up
    barrier()
    e0.record(stream)
    for _ in range(reps):
        lat.copy_(noise)
        ctx.denoise(io, lat, x_txt, 6)
    e1.record(stream)
    barrier()
    d_ms = slowest_rank(e0.elapsed_time(e1), dist) / reps
    e0.record(stream)
    for _ in range(reps):
        lat.copy_(h_noise, non_blocking=True)
        x_txt.copy_(h_txt, non_blocking=True)
        ctx.denoise(io, lat, x_txt, 6)
        h_out.copy_(lat, non_blocking=True)
    e1.record(stream)
    barrier()
    de_ms = slowest_rank(e0.elapsed_time(e1), dist) / reps
    if ctx.sync_status() != 0:
        raise RuntimeError("denoise failed")
    if not bool(torch.isfinite(h_out).all()):
        raise RuntimeError("denoise produced non-finite values")
    in_bytes = h_noise.numel() * 4 + h_txt.numel() * h_txt.element_size()
    return {"ms": round(d_ms / world, 1), "steps": 6, "latent": list(shape),
            "e2e": {"value": round(de_ms / world, 1), "unit": "ms",
                    "h2d_bytes_per_run": in_bytes, "d2h_bytes_per_run": h_out.numel() * 4}}


def sp_fused_timing(ctx, block, ranks: int = 4, reps: int = 3, mx: bool = False) -> dict:
    """One block of the 4096^2 step under Ulysses SP with the fused exchanges,
    all `ranks` ranks on this one GPU: each rank's three stages (RMSNorm +
    QKV storing into every rank's receive buffer; attention of its head group
    storing into every rank's out-projection input; out-projection and FFN)
    through the library, timed per stage with CUDA events, next to the
    unsharded block. On one GPU the ranks run one after another, so the total
    is the block's whole work plus the decomposition's overhead; the per-rank
    stage times are what one GPU of an SP group would spend. With mx the
    context is MXFP8 and the ranks run its MXFP8 block."""
    import torch

    from image_generation_b200.ulysses import FusedUlyssesRank

    n_total = N_TOK
    rs = [FusedUlyssesRank(ctx, r, ranks, n_total, D, H, ctx.cfg.head_dim, F, mx=mx)
          for r in range(ranks)]
    for r in rs:
        r.connect([q.recv.data_ptr() for q in rs], [q.o.data_ptr() for q in rs],
                  [q.o_sf.data_ptr() for q in rs] if mx else None)
    c = torch.empty(D, device="cuda")
    mod = torch.empty(1, 6, D, device="cuda")
    rope = torch.empty(n_total, ctx.cfg.head_dim // 2, 2, device="cuda")
    ctx.time_embed(0.5, c)
    ctx.adaln_project(c, 0, 1, mod)
    ctx.rope_table([(0, GRID, GRID)], N_TXT, rope)
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    x = torch.randn(n_total, D, device="cuda", generator=g)
    xs = [x[r.rows()].clone() for r in rs]
    stages = ("qkv_scatter", "attention_scatter", "finish")
    ev = {s: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(ranks)] for s in stages}
    times = {s: [] for s in stages}
    for rep in range(reps + 1):
        for i, r in enumerate(rs):
            ev["qkv_scatter"][i][0].record()
            r.qkv_scatter(xs[i], mod[0], block, rope[r.rows()])
            ev["qkv_scatter"][i][1].record()
        for i, r in enumerate(rs):
            ev["attention_scatter"][i][0].record()
            r.attention_scatter()
            ev["attention_scatter"][i][1].record()
        for i, r in enumerate(rs):
            ev["finish"][i][0].record()
            r.finish(xs[i], mod[0], block)
            ev["finish"][i][1].record()
        torch.cuda.synchronize()
        if rep:  # the first pass warms up
            for s in stages:
                times[s].append(sum(a.elapsed_time(b) for a, b in ev[s]) / ranks)
    if ctx.sync_status() != 0:
        raise RuntimeError("sequence-parallel stages failed")
    per_rank = {s: round(sorted(v)[len(v) // 2], 3) for s, v in times.items()}
    xt = torch.randn(N_TXT, D, device="cuda", generator=g).bfloat16()
    xi = torch.randn(GRID * GRID, D, device="cuda", generator=g).bfloat16()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx.block_forward(0, 0.5, xi, [(0, GRID, GRID)], xt, mod=mod[0])
    e0.record()
    for _ in range(reps):
        ctx.block_forward(0, 0.5, xi, [(0, GRID, GRID)], xt, mod=mod[0])
    e1.record()
    torch.cuda.synchronize()
    if ctx.sync_status() != 0:
        raise RuntimeError("unsharded block failed")
    return {"ranks": ranks, "tokens": n_total, "ms_per_rank": per_rank,
            "ms_per_rank_total": round(sum(per_rank.values()), 3),
            "ms_unsharded_block": round(e0.elapsed_time(e1) / reps, 3),
            "note": "all ranks on one GPU, one after another; the exchanges are the QKV and "
                    "attention epilogues' stores into the other ranks' buffers"}


def optional_leg(name: str, fn):
    """Run one of the extra measurements; a failure there is reported in its
    field instead of costing the whole line (the step's own timing is not
    guarded)."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001 - reported, not hidden
        print(f"bench: {name} failed: {e}", file=sys.stderr, flush=True)
        return {"error": f"{type(e).__name__}: {str(e).splitlines()[0][:200]}"}


def block_flops(n: int, d) -> float:
    I = d.heads * d.head_dim
    return 8.0 * n * d.hidden * I + 4.0 * n * d.hidden * d.ffn + 4.0 * n * n * I


def run_h3dit(args):
    import torch

    world, rank, local = dist_info()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        dist = None

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    dh = args.head_dim
    ctx, tw, blocks = make_model(dh, seed=1000 + rank)
    x_txt, x_img = tokens(seed=rank)
    grids = [(0, GRID, GRID)]
    ts = timesteps(args.warmup + args.steps)

    for i in range(args.warmup):
        ctx.step(ts[i], x_img, grids, x_txt)
    barrier()
    st = ctx.sync_status()
    if st != 0:
        raise RuntimeError(f"warm-up failed with status {st}")

    clocks = ClockSampler(local)
    clocks.start()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    ctx.profile_begin()
    n0 = ctx.launch_count()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps - 1)]
    e0.record(stream)
    for i in range(args.steps):
        ctx.step(ts[args.warmup + i], x_img, grids, x_txt)
        if i + 1 < args.steps:
            marks[i].record(stream)
    e1.record(stream)
    barrier()
    launches = ctx.launch_count() - n0
    prof = ctx.profile_end()
    clk = clocks.stop()
    elapsed = slowest_rank(e0.elapsed_time(e1), dist)
    st = ctx.sync_status()
    if st != 0:
        raise RuntimeError(f"timed steps failed with status {st}")
    ms_step = elapsed / args.steps
    bounds = [e0] + marks + [e1]
    per_step = sorted(bounds[i].elapsed_time(bounds[i + 1]) for i in range(args.steps))

    # the same step replayed from a CUDA graph (launch overhead removed)
    graph_ms = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            ctx.step(ts[0], x_img, grids, x_txt)
        graph.replay()
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        barrier()
        graph_ms = slowest_rank(e0.elapsed_time(e1), dist) / args.steps
        del graph
        if ctx.sync_status() != 0:
            raise RuntimeError("graph-replayed steps failed")

    # end to end: host (pinned) tokens in, step, tokens back to the host
    e2e = None
    if not args.no_e2e:
        h_txt = torch.empty(x_txt.shape, dtype=x_txt.dtype, pin_memory=True)
        h_img = torch.empty(x_img.shape, dtype=x_img.dtype, pin_memory=True)
        h_txt.copy_(x_txt)
        h_img.copy_(x_img)
        o_txt = torch.empty_like(h_txt, pin_memory=True)
        o_img = torch.empty_like(h_img, pin_memory=True)

        def e2e_step(t):
            x_txt.copy_(h_txt, non_blocking=True)
            x_img.copy_(h_img, non_blocking=True)
            ctx.step(t, x_img, grids, x_txt)
            o_txt.copy_(x_txt, non_blocking=True)
            o_img.copy_(x_img, non_blocking=True)

        e2e_step(ts[0])
        barrier()
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(ts[i])
        e1.record(stream)
        barrier()
        e_ms = slowest_rank(e0.elapsed_time(e1), dist)
        nbytes = (h_txt.numel() + h_img.numel()) * h_txt.element_size()
        e2e = {"value": round(e_ms / args.steps / world, 2), "unit": "ms",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes}
        if ctx.sync_status() != 0:
            raise RuntimeError("end-to-end steps failed")

    denoise = None
    if not args.no_denoise:
        denoise = optional_leg("denoise", lambda: denoise_timing(ctx, x_txt, rank, world, barrier,
                                                                 dist, stream))

    vae = None
    if world == 1 and not args.no_vae:
        vae = optional_leg("vae", vae_timing)

    streaming = None
    if world == 1 and not args.no_streaming:
        streaming = optional_leg("streaming", lambda: streaming_timings(tw, blocks, x_txt, x_img,
                                                                        grids, dh))
        if "error" not in streaming:
            streaming["resident_50"] = {"ms_per_step": round(ms_step, 1), "streamed_blocks": 0,
                                        "h2d_bytes_per_step": 0}

    sp = None
    if world == 1 and not args.no_sp and dh == 96:
        sp = optional_leg("sp_fused", lambda: sp_fused_timing(ctx, blocks[0]))

    line = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        dom = max((k for k in prof if prof[k][1] > 0), key=lambda k: prof[k][0])
        ms_k, cnt_k = prof[dom]
        per = ms_k / cnt_k
        fl = flops_per_launch(dom, N_TOK, dh)
        if fl:
            achieved = fl / per / 1e9
            peak = float(peaks["bf16_tflops_sustained"])
            roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4)}
        else:
            achieved = bytes_per_launch(dom, N_TOK, dh) / per / 1e6
            peak = float(peaks["hbm_gbs"])
            roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved / peak, 4)}
        roof.update({"kernel": dom, "ms_per_launch": round(per, 4), "launches": cnt_k,
                     "peak_source": f"{peak_src} (sustained bf16)" if fl else f"{peak_src} (hbm copy)",
                     "traffic": traffic_for(dom, dh)})
        kernels = {}
        for k, (ms, cnt) in prof.items():
            if cnt == 0:
                continue
            ent = {"ms_total": round(ms, 3), "launches": cnt,
                   "share": round(ms / max(sum(v[0] for v in prof.values()), 1e-9), 4)}
            f = flops_per_launch(k, N_TOK, dh)
            b = bytes_per_launch(k, N_TOK, dh)
            if f:
                ent["tflops"] = round(f / (ms / cnt) / 1e9, 1)
            elif b:
                ent["gbs"] = round(b / (ms / cnt) / 1e6, 1)
            kernels[k] = ent
        value = ms_step / world
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 2),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded, random-init weights N(0,0.02), tokens N(0,1))",
            "config": {"workload": workload_name(dh), "n_blocks": L, "tokens": N_TOK,
                       "head_dim": dh, "global_batch": world,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (~44 GB of weights read per step)"},
            "tflops_step": round(step_flops(N_TOK, dh) / ms_step / 1e9, 1),
            "frac_of_bf16_peak_step": round(step_flops(N_TOK, dh) / ms_step / 1e9 /
                                            float(peaks["bf16_tflops_sustained"]), 4),
            "roofline": roof, "kernels": kernels, "gpu_launches": launches,
            "e2e": e2e, "clocks": clk,
            "step_ms": {"median": round(per_step[len(per_step) // 2], 2),
                        "min": round(per_step[0], 2), "max": round(per_step[-1], 2)},
            "six_step_ms": round(6 * ms_step, 1),
            "denoise_6step": denoise,
            "weight_streaming": streaming,
            "vae_decode_4096": vae,
            "ulysses_sp4_fused_one_gpu": sp,
            "graph_ms_per_step": None if graph_ms is None else round(graph_ms, 2),
        }
        gemm_kinds = ("qkv", "out_proj", "ffn1", "ffn2")
        if all(prof[k][1] for k in gemm_kinds):
            g_ms = sum(prof[k][0] for k in gemm_kinds)
            g_fl = sum(flops_per_launch(k, N_TOK, dh) * prof[k][1] for k in gemm_kinds)
            line["gemm_tflops"] = round(g_fl / g_ms / 1e9, 1)
            line["attention_tflops"] = kernels.get("attention", {}).get("tflops")
        line["frac_of_nominal_bf16"] = {
            "peak_tflops": NOMINAL_BF16_TFLOPS,
            "step": round(line["tflops_step"] / NOMINAL_BF16_TFLOPS, 4),
            "gemm": round(line.get("gemm_tflops", 0.0) / NOMINAL_BF16_TFLOPS, 4),
            "attention": round((line.get("attention_tflops") or 0.0) / NOMINAL_BF16_TFLOPS, 4)}
        if world == 1 and not args.no_configs:
            def per_shape():
                out = block_timings(96)
                out.update(block_timings(128))
                return out
            line["ms_per_block"] = optional_leg("ms_per_block", per_shape)
        if world == 1 and not args.no_cpu_baseline:
            def cpu():
                v, desc, threads, secs = oracle_sample(dh)
                return {"value": round(v, 1), "unit": "ms", "cores": threads, "kind": "oracle",
                        "estimated": True, "sample": desc, "sample_cpu_seconds": round(secs, 1)}

            def cpu_2k():
                b_ms, b_desc, b_threads = oracle_block_2k(dh)
                return {"value": round(b_ms, 1), "unit": "ms per block", "cores": b_threads,
                        "kind": "oracle", "estimated": False, "sample": b_desc}
            line["cpu_baseline"] = optional_leg("cpu_baseline", cpu)
            line["cpu_baseline_block_2k"] = optional_leg("cpu_baseline_block_2k", cpu_2k)
    # the MXFP8 variant (a11), on the same bf16 weights quantized at create
    if not args.no_mxfp8:
        def mxfp8():
            from image_generation_b200 import h3dit as Hb

            cfg_mx = Hb.make_config(D, H, dh, F, L, N_TOK, precision=Hb.H3DIT_PRECISION_MXFP8)
            ctx_mx = Hb.Context(cfg_mx, tw, blocks)
            ms_mx, prof_mx, launches_mx = time_steps(ctx_mx, args.steps, args.warmup, x_img,
                                                     x_txt, grids, barrier, dist)
            sp_mx = None
            if world == 1 and not args.no_sp and dh == 96:
                sp_mx = optional_leg("sp_fused_mxfp8",
                                     lambda: sp_fused_timing(ctx_mx, blocks[0], mx=True))
            ctx_mx.close()
            peaks, peak_src = load_peaks()
            fp8_peak = 2.0 * float(peaks["bf16_tflops_sustained"])
            gemm_kinds = ("qkv", "out_proj", "ffn1", "ffn2")
            gemm_ms = sum(prof_mx[k][0] for k in gemm_kinds)
            gemm_fl = sum(flops_per_launch(k, N_TOK, dh) * prof_mx[k][1] for k in gemm_kinds)
            g_tf = gemm_fl / gemm_ms / 1e9
            return {"ms_per_step": round(ms_mx, 2), "value": round(ms_mx / world, 2), "unit": "ms",
                    "tflops_step": round(step_flops(N_TOK, dh) / ms_mx / 1e9, 1),
                    "gemm_tflops": round(g_tf, 1),
                    "gemm_frac_of_fp8_peak": round(g_tf / fp8_peak, 4),
                    "fp8_peak": fp8_peak,
                    "fp8_peak_source": f"2 x {peak_src} sustained bf16 (nominal fp8:bf16 = 2)",
                    "gemm_frac_of_nominal_fp8": round(g_tf / NOMINAL_FP8_TFLOPS, 4),
                    "kernels": {k: round(v[0] / max(v[1], 1), 4) for k, v in prof_mx.items()
                                if v[1]},
                    "gpu_launches": launches_mx,
                    "ulysses_sp4_fused_one_gpu": sp_mx}
        mx = optional_leg("mxfp8", mxfp8)
        if rank == 0:
            line["mxfp8"] = mx
    if rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.oracle_configs:
        return run_oracle_configs(args)
    if args.only:
        return run_only(args)
    return run_h3dit(args)


if __name__ == "__main__":
    sys.exit(main())
