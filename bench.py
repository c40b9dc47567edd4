#!/usr/bin/env python
"""Benchmark of the displaced-patch UNet layer step on B200: layer-steps/s and latent px/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 3] [--batch B] [--impl ours|reference]

One "step" is one displaced layer step (dfp_step with is_sync = 0) of the
workload: GN1 statistics + corrected merge, GN1 apply + SiLU, halo refresh,
conv3x3, GN2 statistics + merge + apply, Q/K/V projection, displaced attention,
output projection.  The default workload is the largest one that fits a GPU:
the 240x240x640 map of a 3840 px image in 8 row patches.  The run first executes
the synchronous steps of the schedule (untimed), then exactly W displaced
warm-up steps, then K timed displaced steps, each bracketed by CUDA events on the
library's stream; L2 is flushed (a 512 MB write) between timed steps, outside
the events.  With N > 1 (torchrun) every rank runs an independent replica (the
layer step does not shard on one GPU each: replicas only); value = total steps
of all ranks / max over ranks of the summed step time.  Rank 0 prints one JSON
line.

--impl reference times the CPU oracle (numpy fp64) on the host cores instead:
the same metric on the same workload.  Maps up to 64x64 run full steps; on the
larger maps every oracle step is a bounded sample (see oracle_query_sample).

--batch B runs B images per layer step (the classifier-free-guidance batch, B = 2):
a step is still one dfp_step, now over B images; "images_per_s" reports
value * B and the work model counts all B images.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from patch_diffusion_unet_b200 import configs, inputs  # noqa: E402

METRIC = "displaced-patch layer-steps/s & latent px/s on 1 B200; % tensor/HBM roofline"
UNIT = "layer-steps/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--batch", type=int, default=1, help="images per step (2: the guidance batch)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--profile-steps", type=int, default=10)
    ap.add_argument("--min-warmup-s", type=float, default=0.0,
                    help="keep warming up past W steps until this much wall time has passed "
                         "(the line's \"warmup\" then reports the steps actually run)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch each kernel only after its predecessor completed (no programmatic dependent launch)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------- work model

def work_model(cfg):
    """Algorithmic FLOPs / bytes per launch of each kernel of one layer step (all images of
    a batch: every kernel does each image's work once)."""
    B = cfg.get("batch", 1)
    wm = _work_model_one_image(cfg)
    return {k: (v[0], B * v[1]) if isinstance(v, tuple) else (B * v if k == "_total_flops" else v)
            for k, v in wm.items()}


def unet_flops(cfg):
    """Algorithmic FLOPs of one UNet evaluation (2 per multiply-add; the stride-2 convs at
    their own cost, the latent's 4 channels unpadded; the timestep MLP and the norms are
    not counted): {part: FLOPs} and the total."""
    H, W, lat = cfg["H"], cfg["W"], cfg["latent_c"]
    c0, c1, c2 = cfg["widths"]
    T = cfg["ctx_len"]
    L0, L1, L2 = H * W, H * W // 4, H * W // 16

    def conv(L, ci, co):
        return 2.0 * L * 9 * ci * co

    def res(L, ci, co):
        return conv(L, ci, co) + conv(L, co, co) + (2.0 * L * ci * co if ci != co else 0.0)

    def xf(L, c):
        F = 4 * c
        heads = c // 64
        return (2.0 * L * c * 3 * c + 4.0 * L * L * 64 * heads + 2.0 * L * c * c +          # self-attention
                2.0 * L * c * c + 4.0 * L * T * 64 * heads + 2.0 * L * c * c +             # cross-attention
                2.0 * L * c * 2 * F + 2.0 * L * F * c)                                     # GEGLU feed-forward
    parts = {
        "conv_in": conv(L0, lat, c0), "res0": res(L0, c0, c0), "down0": conv(L1, c0, c0),
        "res1": res(L1, c0, c1), "xf1": xf(L1, c1), "down1": conv(L2, c1, c1),
        "res2": res(L2, c1, c2), "xf2": xf(L2, c2), "up1": conv(L1, c2, c2),
        "ures1": res(L1, c2 + c1, c1), "uxf1": xf(L1, c1), "up0": conv(L0, c1, c1),
        "ures0": res(L0, c1 + c0, c0), "conv_out": conv(L0, c0, lat),
    }
    return parts, sum(parts.values())


def _work_model_one_image(cfg):
    H, W, C, N, heads = cfg["H"], cfg["W"], cfg["C"], cfg["n_patches"], cfg["heads"]
    L, d = H * W, cfg["head_dim"]
    e = 2 if cfg["dtype"] == "bf16" else 4
    R = H // N
    if cfg.get("block") == "sdxl_stage":
        F, T = cfg["ffn_inner"], cfg["ctx_len"]
        ln = ("hbm", 2 * L * C * e)
        wm = {
            "norm1 + SiLU + halo (fused)": ("hbm", 2 * L * C * e + 2 * 2 * (N - 1) * W * C * e),
            "conv1 (tcgen05)": ("tensor", 2.0 * L * C * 9 * C),
            "norm2 + SiLU + halo (fused)": ("hbm", 2 * L * C * e + 2 * 2 * (N - 1) * W * C * e),
            "conv2 + residual (tcgen05)": ("tensor", 2.0 * L * C * 9 * C),
            "layernorm 1": ln, "layernorm 2": ln, "layernorm 3": ln,
            "self-attn qkv (tcgen05)": ("tensor", 2.0 * L * C * 3 * C),
            "self-attention (tcgen05)": ("tensor", 4.0 * L * L * d * heads),
            "self-attn out + residual (tcgen05)": ("tensor", 2.0 * L * C * C),
            "cross-attn q (tcgen05)": ("tensor", 2.0 * L * C * C),
            "cross-attention (tcgen05)": ("tensor", 4.0 * L * T * d * heads),
            "cross-attn out + residual (tcgen05)": ("tensor", 2.0 * L * C * C),
            "ff proj + GEGLU (tcgen05)": ("tensor", 2.0 * L * C * 2 * F),
            "ff out + residual (tcgen05)": ("tensor", 2.0 * L * F * C),
        }
        per_block = 2.0 * L * C * 6 * C + 4.0 * L * (L + T) * d * heads + 2.0 * L * C * 3 * F
        wm["_total_flops"] = 2 * 2.0 * L * C * 9 * C + cfg["n_xformer"] * per_block
        wm["_rows_per_patch"] = R
        return wm
    return {
        "gn1 + SiLU + halo (fused)": ("hbm", 2 * L * C * e + 2 * 2 * (N - 1) * W * C * e),
        "conv (tcgen05)": ("tensor", 2.0 * L * C * 9 * C),
        "gn2 (fused)": ("hbm", 2 * L * C * e),
        "qkv (tcgen05)": ("tensor", 2.0 * L * C * 3 * C),
        "attention (tcgen05)": ("tensor", 4.0 * L * L * d * heads),
        "out projection (tcgen05)": ("tensor", 2.0 * L * C * C),
        "_total_flops": 2.0 * L * C * 9 * C + 2.0 * L * C * 4 * C + 4.0 * L * L * d * heads,
        "_rows_per_patch": R,
    }


# ---------------------------------------------------------------------------- ncu traffic

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu capture
# (profiles/), keyed by workload and kernel, with a hash of the kernel's sources at
# capture time: once the kernel changes the figure no longer applies and is reported null.
NCU_TRAFFIC = {
    ("sdxl3840-240x240x640-n8-bf16", "attention (tcgen05)"):
        (516.46e6, ("tc_attention.cu", "dfp_common.cuh", "exp2_poly.cuh"), "ad4f4e3730a65d4a"),
}


def ncu_traffic(workload, kernel):
    ent = NCU_TRAFFIC.get((workload, kernel))
    if ent is None:
        return None
    nbytes, files, sha = ent
    m = hashlib.sha256()
    for fn in files:
        with open(os.path.join(ROOT, "patch_diffusion_unet_b200", "csrc", fn), "rb") as f:
            m.update(f.read())
    return nbytes if m.hexdigest()[:16] == sha else None


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    COLS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
            "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
            "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.COLS}", "--format=csv,noheader,nounits",
                                       "-i", str(gpu_index), "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        for line in self.f.read().splitlines():
            cols = [c.strip() for c in line.split(",")]
            if len(cols) < 9:
                continue
            try:
                sm.append(float(cols[1]))
                mx.append(float(cols[2]))
            except ValueError:
                continue
            for name, v in zip(self.NAMES, cols[5:9]):
                if v == "Active":
                    reasons.add(name)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- CPU oracle leg

def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


def oracle_query_sample(cfg, per_patch=32):
    """Query tokens whose attention the oracle computes in one bounded step.

    Maps up to 64x64 (4096 tokens) run whole steps (None).  On larger maps a whole
    fp64 step is minutes of CPU work (the 240x240 map's attention alone is 8.5 TFLOP
    and 33 G exponentials), so each step computes GroupNorm, conv and the Q/K/V
    projections in full and the attention for `per_patch` evenly spaced query tokens
    of every patch; oracle_step_seconds adds the time of the skipped queries."""
    L = cfg["H"] * cfg["W"]
    if L <= 4096:
        return None
    N = cfg["n_patches"]
    Lp = L // N
    return np.concatenate([p * Lp + np.linspace(0, Lp - 1, per_patch).round().astype(np.int64) for p in range(N)])


def oracle_step_seconds(blk, cfg, x, t, is_sync, sample):
    """Seconds for one oracle layer step.  With a query sample of n of the L tokens the
    step runs with attention for those n queries only; the attention of the other L - n
    queries is accounted by timing the oracle's own softmax_attention on the same n
    queries (per patch and head, against full-length K/V, as the step calls it) and
    scaling that time by (L - n) / n."""
    import oracle
    t0 = time.perf_counter()
    blk.step(x, t, is_sync, **({} if sample is None else {"query_tokens": sample}))
    dt = time.perf_counter() - t0
    if sample is None:
        return dt
    L, heads, N = cfg["H"] * cfg["W"], cfg["heads"], cfg["n_patches"]
    Lp, n = L // N, len(sample)
    extra = 0.0
    for b in getattr(blk, "blocks", [blk]):
        last = b.attn.last
        q, k, v = last["q"], last["k"], last["v"]
        d = q.shape[1] // heads
        t1 = time.perf_counter()
        for p in range(N):
            sel = sample[(sample >= p * Lp) & (sample < (p + 1) * Lp)]
            for h in range(heads):
                c = slice(h * d, (h + 1) * d)
                oracle.softmax_attention(q[sel, c], k[:, c], v[:, c], 1.0 / np.sqrt(d))
        extra += (time.perf_counter() - t1) * (L - n) / n
    return dt + extra


def oracle_sample_text(cfg, sample):
    if sample is None:
        return "full UNet evaluations" if cfg.get("block") == "unet" else "full layer steps"
    L = cfg["H"] * cfg["W"]
    return (f"bounded steps: GroupNorms, conv and Q/K/V/O projections in full, attention output for "
            f"{len(sample)} of {L} query tokens ({len(sample) // cfg['n_patches']} evenly spaced per patch); "
            f"the other queries' attention time added from the oracle's softmax_attention timed on the "
            f"same queries, scaled by (L - n) / n")


def oracle_displaced_rate(cfg, n_disp=2):
    """Time the oracle as it stands on displaced steps of the workload (after one sync step)."""
    import oracle
    wl = inputs.SyntheticWorkload(cfg)
    blk = oracle.make_block(cfg, wl.weights, wl.context)
    sample = oracle_query_sample(cfg)
    oracle_step_seconds(blk, cfg, wl.x(0), 0, 1, sample)
    dt = 0.0
    w0 = time.perf_counter()
    for t in range(1, 1 + n_disp):
        dt += oracle_step_seconds(blk, cfg, wl.x(t), t, 0, sample)
    wall = time.perf_counter() - w0
    return n_disp / dt, _oracle_threads(), wall, sample


# ---------------------------------------------------------------------------- main

def replica_throughput(local_ms, units, world, device):
    """Whole-job rate over `world` replicas: every rank's timed region is reduced to the
    maximum over ranks (the slowest replica bounds the job) and all ranks' units count.
    Returns (units per second, max milliseconds)."""
    import torch
    t = torch.tensor([float(local_ms)], device=device, dtype=torch.float64)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_ms = float(t.item())
    return world * units / (max_ms / 1e3), max_ms


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return world, rank, local


def workload_config(cfg, B):
    """The keys of a line's `config` that name the workload, the same in both arms."""
    if cfg["block"] == "unet":
        return {"workload": cfg["name"], "H": cfg["H"], "W": cfg["W"], "widths": list(cfg["widths"]),
                "n_patches": cfg["n_patches"], "step": "displaced UNet evaluation (is_sync=0)"}
    return {"workload": cfg["name"], "H": cfg["H"], "W": cfg["W"], "C": cfg["C"], "n_patches": cfg["n_patches"],
            "heads": cfg["heads"], "batch": B, "step": "displaced (is_sync=0)"}


def run_reference(args, cfg):
    """The reference arm: the oracle on the host cores, rank 0 only, on the same workload,
    metric and unit; the synchronous steps of the schedule, then W displaced warm-up steps
    and K timed displaced steps, each bounded as oracle_step_seconds says."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    B = cfg.get("batch", 1)
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    wl = inputs.SyntheticWorkload(cfg)
    n_sync = cfg["n_sync"]
    if cfg["block"] == "unet":
        # the oracle UNet, whole steps (one UNet evaluation each) at the DDIM timesteps
        from oracle import unet_oracle
        net = unet_oracle.DisplacedUNet(cfg, wl.weights, wl.context)
        taus, x = ddim_taus(cfg), wl.latent()
        sample = None

        def run(t, is_sync):
            t0 = time.perf_counter()
            net.step(x, t, is_sync, taus[t % len(taus)])
            return time.perf_counter() - t0
    else:
        blk = oracle.make_block(cfg, wl.weights, wl.context)
        sample = oracle_query_sample(cfg)

        def run(t, is_sync):
            return oracle_step_seconds(blk, cfg, wl.x(t), t, is_sync, sample)
    t = 0
    for t in range(n_sync):
        run(t, 1)
    for _ in range(args.warmup):
        t += 1
        run(t, 0)
    dt = 0.0
    for _ in range(args.steps):
        t += 1
        dt += run(t, 0)
    threads = _oracle_threads()
    value = args.steps / dt
    L = cfg["H"] * cfg["W"]
    unit = "unet-steps/s" if cfg["block"] == "unet" else UNIT
    what = "displaced UNet evaluations" if cfg["block"] == "unet" else "displaced layer steps"
    text = f"{args.steps} {what} after {n_sync} sync and {args.warmup} warm-up steps; " + \
        oracle_sample_text(cfg, sample)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "latent_px_per_s": value * L * B, "images_per_s": value * B,
        "config": {**workload_config(cfg, B), "parallelism": "rank 0 on the host cores", "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": text},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def ddim_taus(cfg, n_steps=50):
    """The DDIM timesteps visited, largest first: (n - 1 - k) n_train / n + 1."""
    ratio = cfg["ddim_train_steps"] // n_steps
    return [(n_steps - 1 - k) * ratio + 1 for k in range(n_steps)]


def oracle_unet_rate(cfg):
    """The oracle UNet on the host cores: one displaced step after one synchronous step."""
    from oracle import unet_oracle
    wl = inputs.SyntheticWorkload(cfg)
    net = unet_oracle.DisplacedUNet(cfg, wl.weights, wl.context)
    taus = ddim_taus(cfg)
    x = wl.latent()
    net.step(x, 0, 1, taus[0])
    t0 = time.perf_counter()
    net.step(x, 1, 0, taus[1])
    dt = time.perf_counter() - t0
    return 1.0 / dt, _oracle_threads(), dt


def run_unet(args, cfg):
    """The multi-level UNet: a step is one displaced UNet evaluation (dfp_step at a DDIM
    timestep); e2e is a whole DDIM run through dfp_ddim_sample with the starting latent
    copied in from pinned host memory and the result copied out inside the timed region."""
    import torch
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    import torch.distributed as dist
    from patch_diffusion_unet_b200 import dfp
    H, W = cfg["H"], cfg["W"]
    wl = inputs.SyntheticWorkload(cfg)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(dict(wl.weights, context=wl.context))
    blk.set_launch_overlap(not args.no_overlap)
    stream = blk.stream
    rng = np.random.default_rng(1)
    xs = [inputs.to_torch(inputs.round_to(rng.standard_normal((H, W, cfg["latent_c"])), "bf16"), "bf16").cuda()
          for _ in range(4)]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    taus = ddim_taus(cfg)

    def step(t, is_sync):
        blk.set_timestep(taus[t % len(taus)])
        blk.step(xs[t % len(xs)], t, is_sync)

    for t in range(cfg["n_sync"]):
        step(t, 1)
    t = cfg["n_sync"] - 1
    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local] if \
        os.environ.get("CUDA_VISIBLE_DEVICES") else str(local)
    sampler = ClockSampler(gpu_index)
    for _ in range(args.warmup):
        t += 1
        step(t, 0)
        flush.zero_()
    blk.check_device()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        t += 1
        ev[i][0].record(stream)
        step(t, 0)
        ev[i][1].record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    blk.check_device()
    value, total_ms_max = replica_throughput(float(sum(a.elapsed_time(b) for a, b in ev)), args.steps, world, "cuda")
    launches = blk.launches_per_step()
    # per-kernel time shares (kernel names repeat across layers: summed per name and step)
    blk.set_profiling(True)
    per = {}
    for _ in range(args.profile_steps):
        t += 1
        step(t, 0)
        sums = {}
        for name, ms in blk.kernel_times():
            sums[name] = sums.get(name, 0.0) + ms
        for k, v in sums.items():
            per.setdefault(k, []).append(v)
        flush.zero_()
    blk.set_profiling(False)
    kern_us = {k: 1e3 * statistics.mean(v) for k, v in per.items()}
    # end to end: a DDIM run of the whole schedule through the public entry point
    e2e = None
    if not args.no_e2e:
        n_steps = 50
        xh = torch.from_numpy(np.ascontiguousarray(wl.latent(), np.float32)).pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        xd = torch.empty_like(xh, device="cuda")
        for rep in range(2):   # the first run warms up
            torch.cuda.synchronize()
            w0 = time.perf_counter()
            with torch.cuda.stream(stream):
                xd.copy_(xh, non_blocking=True)
            out = blk.ddim_sample(xd, n_steps, cfg["n_sync"], cfg["ddim_train_steps"], cfg["beta_start"],
                                  cfg["beta_end"])
            with torch.cuda.stream(stream):
                yh.copy_(out, non_blocking=True)
            blk.synchronize()
            e_total = time.perf_counter() - w0
        e2e_rate, _ = replica_throughput(e_total * 1e3, n_steps, world, "cuda")
        nbytes = H * W * cfg["latent_c"] * 4
        e2e = {"value": e2e_rate, "unit": "unet-steps/s", "h2d_bytes_per_step": nbytes / n_steps,
               "d2h_bytes_per_step": nbytes / n_steps, "steps": n_steps,
               "api": "dfp_ddim_sample (50 DDIM steps, first n_sync synchronous), latent in and out through pinned host memory, wall clock",
               "images_per_s": e2e_rate / n_steps}
    pk, pk_src = peaks()
    parts, total = unet_flops(cfg)
    ms_step = total_ms_max / args.steps
    ach = total / (ms_step * 1e-3) / 1e12
    peak = pk.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    roof = {"kernel": "whole UNet step", "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": ach / peak, "traffic": None, "peak_source": f"{pk_src} bf16 burst", "work_per_launch": total,
            "us_per_launch": 1e3 * ms_step}
    blk.close()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, dt = oracle_unet_rate(cfg)
        cpu = {"value": rate, "unit": "unet-steps/s", "cores": threads, "kind": "oracle",
               "sample": f"1 displaced UNet step of {cfg['name']} after 1 sync step ({dt:.1f} s)"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "unet-steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random weights, random latents)",
            "latent_px_per_s": value * H * W, "tensor_tflops_per_step": ach,
            "config": {**workload_config(cfg, 1), "parallelism": f"replicas{world}",
                       "l2": "flushed between timed steps (512 MB write, outside the events)"},
            "gpu_launches": launches * args.steps, "launches_per_step": launches,
            "kernels_us": {k: round(v, 2) for k, v in kern_us.items()},
            "flops_per_part_g": {k: round(v / 1e9, 2) for k, v in parts.items()},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    cfg = configs.get(args.config)
    B = max(1, args.batch)
    if B > 1:
        cfg = configs.get(cfg, batch=B, name=f"{cfg['name']}-b{B}")
    if args.impl == "reference":
        return run_reference(args, cfg)
    if cfg["block"] == "unet":
        return run_unet(args, cfg)

    import torch
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    import torch.distributed as dist
    from patch_diffusion_unet_b200 import dfp

    dtype = cfg["dtype"]
    L = cfg["H"] * cfg["W"]
    wl = inputs.SyntheticWorkload(cfg)
    blk = dfp.DisplacedPatchBlock(cfg)
    blk.load_weights(dict(wl.weights, context=wl.context) if wl.context is not None else wl.weights)
    blk.set_launch_overlap(not args.no_overlap)
    stream = blk.stream
    # a pool of distinct inputs (the steps cycle through it); fewer of the large maps
    n_pool = 16 if L <= 16384 else 4
    host_x = [inputs.to_torch(wl.x(t), dtype) for t in range(n_pool)]
    xs = [h.cuda() for h in host_x]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")

    def x_of(t):
        return xs[t % n_pool]

    n_sync = cfg["n_sync"]
    for t in range(n_sync):
        blk.step(x_of(t), t, 1)
    t = n_sync - 1
    # warm-up: exactly W displaced steps (more only if --min-warmup-s asks for a minimum time)
    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local] if \
        os.environ.get("CUDA_VISIBLE_DEVICES") else str(local)
    sampler = ClockSampler(gpu_index)
    w_start = time.perf_counter()
    n_warm = 0
    while n_warm < args.warmup or time.perf_counter() - w_start < args.min_warmup_s:
        t += 1
        blk.step(x_of(t), t, 0)
        flush.zero_()
        n_warm += 1
        if n_warm % 16 == 0:
            torch.cuda.synchronize()
    blk.check_device()

    # ---- timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    wall0 = time.perf_counter()
    for i in range(args.steps):
        t += 1
        ev[i][0].record(stream)
        blk.step(x_of(t), t, 0)
        ev[i][1].record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    blk.check_device()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    value, total_ms_max = replica_throughput(float(sum(step_ms)), args.steps, world, "cuda")
    launches = blk.launches_per_step()

    # ---- per-kernel durations (separate profiled steps, same stream, L2 flushed between)
    blk.set_profiling(True)
    per = {}
    for _ in range(args.profile_steps):
        t += 1
        blk.step(x_of(t), t, 0)
        for name, ms in blk.kernel_times():
            per.setdefault(name, []).append(ms)
        flush.zero_()
    blk.set_profiling(False)
    kern_us = {k: 1e3 * statistics.mean(v) for k, v in per.items()}

    # ---- sync steps (every patch fresh), timed the same way, for context
    n_sync_t = min(args.steps, 50)
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_sync_t)]
    for i in range(n_sync_t):
        t += 1
        sev[i][0].record(stream)
        blk.step(x_of(t), t, 1)
        sev[i][1].record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    sync_ms = statistics.mean(a.elapsed_time(b) for a, b in sev)

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        # the pipelined host-buffer API as a serving loop would drive it: every step copies
        # its input from pinned host memory and its output back, overlapped with the
        # neighbouring steps' kernels; L2 is still flushed between steps, on the step's
        # stream and inside the timed region
        xh = [h.pin_memory() for h in host_x]
        yh = [torch.empty(B * L, cfg["C"], dtype=xh[0].dtype).pin_memory() for _ in range(2)]
        for i in range(4):
            t += 1
            blk.step_host_async(xh[t % n_pool], yh[i & 1], t, 0)
        blk.synchronize()
        n_e = max(10, min(args.steps, 100))
        torch.cuda.synchronize()
        w0 = time.perf_counter()
        for i in range(n_e):
            t += 1
            blk.step_host_async(xh[t % n_pool], yh[i & 1], t, 0)
            with torch.cuda.stream(stream):
                flush.zero_()
        blk.synchronize()
        e_total = time.perf_counter() - w0
        e2e_rate, _ = replica_throughput(e_total * 1e3, n_e, world, "cuda")
        nbytes = B * L * cfg["C"] * (2 if dtype == "bf16" else 4)
        e2e = {"value": e2e_rate, "unit": UNIT, "h2d_bytes_per_step": nbytes,
               "d2h_bytes_per_step": nbytes, "steps": n_e,
               "api": "dfp_step_host_async (pinned host buffers) + dfp_synchronize, wall clock",
               "l2": "flushed between steps inside the timed region"}

    # ---- roofline of the dominant kernel
    pk, pk_src = peaks()
    wm = work_model(cfg)
    dom = max(kern_us, key=kern_us.get) if kern_us else None
    roof = None
    if dom and dom in wm:
        bound, work = wm[dom]
        us = kern_us[dom]
        if bound == "tensor":
            ach = work / (us * 1e-6) / 1e12
            peak = pk.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
            roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                    "frac": ach / peak, "traffic": ncu_traffic(cfg["name"], dom),
                    "peak_source": f"{pk_src} bf16 burst",
                    "work_per_launch": work, "us_per_launch": us}
        else:
            ach = work / (us * 1e-6) / 1e9
            peak = pk.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
            roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak, "traffic": ncu_traffic(cfg["name"], dom),
                    "peak_source": f"{pk_src} HBM copy",
                    "work_per_launch": work, "us_per_launch": us}

    blk.close()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, threads, wall, sample = oracle_displaced_rate(cfg)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"2 displaced layer steps of {cfg['name']} after 1 sync step ({wall:.1f} s wall); " +
                         oracle_sample_text(cfg, sample)}

    if rank == 0:
        ms_step = total_ms_max / args.steps
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": n_warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if dtype == "bf16" else "f32", "data": "synthetic",
            "latent_px_per_s": value * L * B, "images_per_s": value * B,
            "tensor_tflops_per_step": wm["_total_flops"] / (ms_step * 1e-3) / 1e12,
            "config": {**workload_config(cfg, B), "launch_overlap": not args.no_overlap,
                       "parallelism": f"replicas{world}",
                       "l2": "flushed between timed steps (512 MB write, outside the events)"},
            "sync_ms_per_step": sync_ms,
            "gpu_launches": launches * args.steps,
            "launches_per_step": launches,
            "kernels_us": {k: round(v, 2) for k, v in kern_us.items()},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
