#!/usr/bin/env python
"""Benchmark of the DiT denoiser forward on B200.

Workload (one "step" = one whole forward): DiT-XL/2 with classifier-free guidance at
256 px — 16 latents 4x32x32, duplicated to 32 rows (labels [y; null]), patch 2 ->
256 tokens per row, d = 1152, 28 blocks, 16 heads, guidance s = 1.5 on all channels,
seeded N(0, 0.02) weights, synthetic inputs.  8192 tokens per step per GPU.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one replica per GPU (weak scaling, no collective on the data path) under
torch.distributed.run.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dit_synth as S  # noqa: E402

METRIC = "DiT-XL/2 bf16 fwd tokens/sec on 1 B200; % of dense BF16 tensor peak"
CFG = S.DIT_XL2_CFG256
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of each kernel kind,
# from one cold-cache ncu capture of this workload; a kind whose kernel has changed since its
# capture has no entry (the roofline then reports traffic null).
TRAFFIC_BYTES = {"fc1": 55.16e6, "fc2": 130.17e6, "qkv": 44.23e6, "proj": 59.56e6, "attn": 65.21e6,
                 "ln": 38.14e6, "adaln": 473.41e6, "decode": 18.97e6}
TRAFFIC_SOURCE = "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --clock-control none, one launch, cold cache"
# fallback peaks (used only when MEASURED_PEAKS.json is absent)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0
KINDS = ["cond", "adaln", "patch", "ln", "qkv", "attn", "proj", "fc1", "fc2", "decode", "sampler"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


WORKLOADS = {
    "xl2_256": S.DIT_XL2_CFG256,           # the headline workload
    "xl2_512": S.DIT_XL2_CFG512,
    "video": S.VIDEO_RF,
    "b4": S.DIT_B4_BF16,
    "xl2_256_fp8": S.DIT_XL2_CFG256.with_(ffn_fp8=1),
    "xl2_256_fp8all": S.DIT_XL2_CFG256.with_(ffn_fp8=1, attn_fp8=1),
}


def fp8_desc(cfg):
    parts = [n for n, on in (("attention projections", getattr(cfg, "attn_fp8", 0)),
                              ("feed-forward", getattr(cfg, "ffn_fp8", 0))) if on]
    return " + ".join(parts)


def workload_desc(cfg):
    lat = (f"{cfg.in_channels}x{cfg.frames}x{cfg.height}x{cfg.width}" if cfg.frames > 1
           else f"{cfg.in_channels}x{cfg.height}x{cfg.width}")
    extra = f", FP8 E4M3 {fp8_desc(cfg)}" if fp8_desc(cfg) else ""
    return (f"{cfg.name}: {cfg.batch} latents {lat} -> {cfg.rows} rows x {cfg.tokens} tokens, d={cfg.hidden}, "
            f"{cfg.depth} blocks, {cfg.heads} heads, s={cfg.cfg_scale}{extra}")


def kernel_flops(cfg):
    """Algorithmic FLOPs (2 per multiply-add) per launch of each kernel kind, and per step.
    Tokens inside the blocks include the in-context design's two condition tokens; the
    embedding and the decoder count the patch tokens only."""
    R, T, d, mlp, H = cfg.rows, cfg.tokens, cfg.hidden, cfg.mlp_hidden, cfg.heads
    Ts = getattr(cfg, "seq_tokens", T)
    dh = cfg.head_dim
    M = R * Ts
    mpb = getattr(cfg, "mod_per_block", 6)
    nmod = (mpb * cfg.depth + 2) * d if mpb else 0
    cross = getattr(cfg, "block_kind", 0) == S.BLOCK_CROSS_ATTN
    per = {
        "cond": 2 * R * (cfg.freq_dim * d + d * d),
        "adaln": 2 * R * nmod * d + (2 * (2 * R) * (2 * d * cfg.depth) * d if cross else 0),
        "patch": 2 * R * T * d * cfg.patch_dim,
        "qkv": 2 * M * 3 * d * d,
        "attn": 4 * R * H * Ts * Ts * dh + (2 * M * d * d + 8 * M * d if cross else 0),
        "proj": 2 * M * d * d + (2 * M * d * d if cross else 0),
        "fc1": 2 * M * mlp * d,
        "fc2": 2 * M * d * mlp,
        "decode": 2 * R * T * d * cfg.out_dim,
        "ln": 0,
    }
    step = (per["cond"] + per["adaln"] + per["patch"] + per["decode"] +
            cfg.depth * (per["qkv"] + per["attn"] + per["proj"] + per["fc1"] + per["fc2"]))
    if cross:   # attn and proj each hold two launches per block: report per launch
        per["attn"] = None
        per["proj"] = None
    return per, step


def ln_bytes(cfg):
    M = cfg.rows * cfg.tokens
    return M * cfg.hidden * (4 + 2)  # read f32 residual, write bf16


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, polled through NVML every 20 ms in a
    background thread while the timed region runs (the fields of nvidia-smi's clocks query)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, index: int, period_s: float = 0.02):
        self.index = index
        self.period = period_s
        self.rows = []
        self.max_mhz = None
        self._stop = threading.Event()
        self.thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
            return
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def _poll(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.rows.append((sm, pw, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in self.rows if r[1] > 200.0] or self.rows
        reasons = set()
        for _, _, rs in self.rows:
            for name, attr in self.REASONS:
                if rs & getattr(self.nv, attr, 0):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[1] for r in self.rows), "source": "NVML, 20 ms polling during the timed region"}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def replica_seed(cfg, rank: int) -> int:
    """Input seed of replica `rank`: the workload's seed + rank, so every replica denoises its
    own latents (weak scaling, no data shared between ranks)."""
    return S.inputs_seed(cfg) + rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of a per-rank float over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    tt = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def aggregate_rate(units_per_rank_step: float, world: int, steps: int, seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank_step * world * steps / seconds


def run_reference(args):
    """The oracle (float64 numpy on the host cores) on a bounded sample per step."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    from oracle import dit_oracle as O
    from threadpoolctl import threadpool_info
    cfg = CFG
    W = S.weight_dict(cfg, S.make_weights(cfg))
    inp = S.make_inputs(cfg)
    x, t, y = inp["x"][:1], inp["t"][:1], inp["y"][:1]
    tokens = 2 * cfg.tokens  # one guided latent = 2 rows
    for _ in range(args.warmup):
        O.forward(cfg, W, x, t, y)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.forward(cfg, W, x, t, y)
    el = time.perf_counter() - t0
    cores = sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas") or os.cpu_count()
    value = tokens * args.steps / el
    sample = "one guided latent (2 rows x 256 tokens, all 28 blocks) per step, float64 numpy oracle"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "global_batch": 1, "rows": 2, "tokens_per_step": tokens},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(cfg, weights):
    """The oracle as it stands, timed on one guided latent (a bounded sample)."""
    from oracle import dit_oracle as O
    from threadpoolctl import threadpool_info
    W = S.weight_dict(cfg, weights)
    inp = S.make_inputs(cfg)
    t0 = time.perf_counter()
    O.forward(cfg, W, inp["x"][:1], inp["t"][:1], inp["y"][:1])
    el = time.perf_counter() - t0
    cores = sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas") or os.cpu_count()
    return {"value": 2 * cfg.tokens / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"one guided latent (2 rows x {cfg.tokens} tokens, all {cfg.depth} blocks), "
                      f"float64 numpy oracle, {el:.1f} s"}


def time_config(cfg, steps, warmup, graph, flush, options=None):
    """Device time of `steps` whole forwards of `cfg` (seeded weights and inputs, L2 flushed between
    steps outside the events), with library options {option: value}.  Returns per-step milliseconds."""
    import torch
    from diffusion_transformer_denoiser_dit_b200 import DiT
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_OPT_USE_GRAPH
    model = DiT(cfg, S.make_weights(cfg))
    model.set_option(DIT_OPT_USE_GRAPH, 1 if graph else 0)
    for opt, val in (options or {}).items():
        model.set_option(opt, val)
    inp = S.make_inputs(cfg)
    x, t, y = (torch.from_numpy(inp[k]).cuda() for k in ("x", "t", "y"))
    out = torch.empty(cfg.out_shape(), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        model.forward(x, t, y, cfg.cfg_scale, out=out, stream=stream)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        model.forward(x, t, y, cfg.cfg_scale, out=out, stream=stream)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    status = model.sync_status()
    model.close()
    if status != 0:
        raise RuntimeError(f"device status {status} while timing {cfg}")
    return [a.elapsed_time(b) for a, b in evs]


def gemm_reference(cfg, kernels, flush, reps=10):
    """cuBLAS (torch.matmul, bf16 in and out, no fused epilogue) on the four block GEMM shapes of
    this workload, timed like the kernel table: CUDA events around each launch, L2 flushed between
    launches.  For context beside the fused kernels; it is not part of the forward."""
    import torch
    M, d = cfg.rows * cfg.tokens, cfg.hidden
    mlp = cfg.mlp_hidden if getattr(cfg, "mlp_hidden", 0) else 4 * d
    shapes = {"qkv": (M, 3 * d, d), "proj": (M, d, d), "fc1": (M, mlp, d), "fc2": (M, d, mlp)}
    out = {}
    g = torch.Generator(device="cuda").manual_seed(0)
    for kind, (m, n, k) in shapes.items():
        a = torch.randn(m, k, device="cuda", generator=g).to(torch.bfloat16)
        w = (torch.randn(n, k, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        y = torch.empty(m, n, device="cuda", dtype=torch.bfloat16)
        for _ in range(3):
            torch.matmul(a, w.t(), out=y)
        ts = []
        for i in range(reps):
            flush.fill_(float(i))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, w.t(), out=y)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        us = statistics.median(ts)
        row = {"shape_mnk": [m, n, k], "cublas_us": us, "cublas_tflops": 2.0 * m * n * k / (us * 1e-6) / 1e12}
        if kind in kernels:
            row["fused_us"] = kernels[kind]["us_per_launch"]
            row["fused_over_cublas"] = kernels[kind]["us_per_launch"] / us
        out[kind] = row
        del a, w, y
    return out


def all_configs(steps, warmup, graph, flush, peak_tf):
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_OPT_PAIR_GEMM
    res = {}
    runs = []
    pair_after = {"c3 XL/2 CFG 256px": "c3 XL/2 CFG 256px, SM-pair GEMMs",
                  "c4 XL/2 CFG 512px": "c4 XL/2 CFG 512px, SM-pair GEMMs"}
    for name, cfg in (("c1 S/8 fp32", S.DIT_S8_F32), ("c2 B/4 bf16", S.DIT_B4_BF16),
                      ("c3 XL/2 CFG 256px", S.DIT_XL2_CFG256), ("c4 XL/2 CFG 512px", S.DIT_XL2_CFG512),
                      ("c5 video RF 4096 tokens", S.VIDEO_RF),
                      ("c3 XL/2 CFG 256px, in-context conditioning", S.DIT_XL2_CFG256.with_(block_kind=S.BLOCK_IN_CONTEXT)),
                      ("c3 XL/2 CFG 256px, cross-attention conditioning", S.DIT_XL2_CFG256.with_(block_kind=S.BLOCK_CROSS_ATTN)),
                      ("c3 XL/2 CFG 256px, adaLN conditioning", S.DIT_XL2_CFG256.with_(block_kind=S.BLOCK_ADALN)),
                      ("c3 XL/2 CFG 256px, FP8 E4M3 feed-forward", S.DIT_XL2_CFG256.with_(ffn_fp8=1)),
                      ("c5 video RF 4096 tokens, FP8 E4M3 feed-forward", S.VIDEO_RF.with_(ffn_fp8=1)),
                      ("c3 XL/2 CFG 256px, FP8 E4M3 attention projections + feed-forward",
                       S.DIT_XL2_CFG256.with_(ffn_fp8=1, attn_fp8=1))):
        runs.append((name, cfg, None))
        if name in pair_after:   # the same workload on SM-pair GEMMs, timed right after it
            runs.append((pair_after[name], cfg, {DIT_OPT_PAIR_GEMM: 1}))
    for name, cfg, opts in runs:
        ms = time_config(cfg, steps, warmup, graph, flush, opts)
        med = statistics.median(ms)
        _, fl = kernel_flops(cfg)
        tf = fl / (med / 1e3) / 1e12
        res[name] = {"ms_per_step_median": med, "ms_per_step_min": min(ms),
                     "tokens_per_s": cfg.rows * cfg.tokens / (med / 1e3),
                     "samples_per_s": cfg.batch / (med / 1e3), "tflops": tf,
                     "frac_of_burst_bf16": tf / peak_tf if cfg.dtype == S.DTYPE_BF16 else None,
                     "dtype": (f"bf16 + e4m3 {fp8_desc(cfg)}" if fp8_desc(cfg) else "bf16")
                              if cfg.dtype == S.DTYPE_BF16 else "f32",
                     "rows": cfg.rows, "tokens_per_row": cfg.tokens, "flops_per_step": fl}
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every kernel directly instead of replaying a CUDA graph")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="xl2_256",
                    help="the workload one step runs (default: the headline DiT-XL/2 CFG 256px; the others are "
                         "for profiling and comparison)")
    ap.add_argument("--pair-gemm", action="store_true", help="run the block GEMMs on SM pairs (DIT_OPT_PAIR_GEMM)")
    ap.add_argument("--lean", action="store_true",
                    help="warm-up and timed steps only (no kernel table, end-to-end or sampler passes): the command "
                         "profiler captures run under")
    ap.add_argument("--all-configs", action="store_true",
                    help="also time the other workloads (S/8 fp32, B/4, XL/2 512px CFG, video) and report them under "
                         "'all_configs' in the same JSON line")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from diffusion_transformer_denoiser_dit_b200 import DiT
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_OPT_PAIR_GEMM, DIT_OPT_REPEAT_KIND, DIT_OPT_USE_GRAPH

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    cfg = WORKLOADS[args.workload]
    weights = S.make_weights(cfg)
    model = DiT(cfg, weights)
    model.set_option(DIT_OPT_USE_GRAPH, 0 if args.no_graph else 1)
    if args.pair_gemm:
        model.set_option(DIT_OPT_PAIR_GEMM, 1)
    inp = S.make_inputs(cfg, seed=replica_seed(cfg, rank))
    x = torch.from_numpy(inp["x"]).cuda()
    t = torch.from_numpy(inp["t"]).cuda()
    y = torch.from_numpy(inp["y"]).cuda()
    out = torch.empty(cfg.out_shape(), dtype=torch.float32, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        model.forward(x, t, y, cfg.cfg_scale, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if model.sync_status() != 0:
        raise RuntimeError("device status error during warm-up")

    sampler = ClockSampler(local)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))          # L2 flush between timed steps (outside the events)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms_median, ms_min = statistics.median(step_ms), min(step_ms)
    total_ms = max_over_ranks(sum(step_ms), world, "cuda")
    status = model.sync_status()
    clocks = sampler.summary()

    if args.lean:
        line = {"metric": METRIC, "value": aggregate_rate(cfg.rows * cfg.tokens, world, args.steps, total_ms / 1e3),
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "config": {"workload": workload_desc(cfg)}, "lean": True, "device_status": status}
        if rank == 0:
            print(json.dumps(line), flush=True)
        model.close()
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    # launches per step of each kernel kind (one profiled forward)
    model.profile(True)
    step()
    torch.cuda.synchronize()
    model.profile(False)
    uses = {k: v[1] for k, v in model.profile_read().items() if v[1] > 0}

    # each kind's own device duration: CUDA events around that kind's launches only (graph
    # bypassed; every other kernel keeps its programmatic-dependent-launch overlap)
    kernels = {}
    n_ev = max(5, min(args.steps, 20))
    for kind, n_use in uses.items():
        model.profile(True, kind)
        for i in range(n_ev):
            flush.fill_(float(i))
            step()
        torch.cuda.synchronize()
        model.profile(False)
        ms, cnt = model.profile_read()[kind]
        kernels[kind] = {"launches_per_step": n_use, "us_per_launch": ms / max(cnt, 1) * 1e3, "ms_per_step": ms / n_ev}

    # Marginal in-pipeline cost of each kind, by differencing: the step time with every kernel
    # of one kind launched twice, minus the plain step time, over the kind's launches per step
    # (CUDA events around whole steps; nothing is inserted between kernels).  A repeated kernel
    # finds its inputs in L2 and a longer step draws more power, so this is a second opinion
    # beside the event durations, not the roofline's timing.
    n_diff = max(10, min(args.steps, 30))

    def median_step_ms(n):
        e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            flush.fill_(float(i))
            e[i][0].record(stream)
            step()
            e[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in e)

    for _ in range(2):
        step()
    for kind, n_use in uses.items():
        base0 = median_step_ms(n_diff)
        model.set_option(DIT_OPT_REPEAT_KIND, KINDS.index(kind))
        for _ in range(2):            # direct run, then graph capture of the doubled forward
            step()
        rep = median_step_ms(n_diff)
        model.set_option(DIT_OPT_REPEAT_KIND, -1)
        for _ in range(2):
            step()
        base1 = median_step_ms(n_diff)
        kernels[kind]["marginal_us_per_launch"] = max(rep - 0.5 * (base0 + base1), 0.0) / n_use * 1e3
    torch.cuda.synchronize()

    # end to end through the host entry point (pinned host buffers, copies inside)
    xh = torch.from_numpy(inp["x"]).pin_memory()
    th = torch.from_numpy(inp["t"]).pin_memory()
    yh = torch.from_numpy(inp["y"]).pin_memory()
    oh = torch.empty(cfg.out_shape(), dtype=torch.float32).pin_memory()
    for _ in range(2):
        model.forward_host_ptr(xh.data_ptr(), th.data_ptr(), yh.data_ptr(), cfg.batch, cfg.cfg_scale, oh.data_ptr())
    e2e_s = 0.0
    for i in range(args.steps):
        flush.fill_(float(i))
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        model.forward_host_ptr(xh.data_ptr(), th.data_ptr(), yh.data_ptr(), cfg.batch, cfg.cfg_scale, oh.data_ptr())
        e2e_s += time.perf_counter() - t0
    e2e_s = max_over_ranks(e2e_s, world, "cuda")

    # sampler loop: forward + fused DDIM update per step, the whole loop replayed as one graph
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_SAMPLER_DDIM
    n_s = 10
    levels = np.linspace(0.05, 0.95, n_s + 1).astype(np.float32)
    mt = np.linspace(950.0, 50.0, n_s).astype(np.float32)
    xs = x.clone()
    for _ in range(3):
        xs.copy_(x)
        model.sample(DIT_SAMPLER_DDIM, xs, y, cfg.cfg_scale, mt, levels, stream=stream)
    torch.cuda.synchronize()
    reps = max(1, args.steps // n_s)
    s_ms = 0.0
    for r in range(reps):
        xs.copy_(x)
        flush.fill_(float(r))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        model.sample(DIT_SAMPLER_DDIM, xs, y, cfg.cfg_scale, mt, levels, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        s_ms += e0.elapsed_time(e1)
    model.profile(True)
    xs.copy_(x)
    model.sample(DIT_SAMPLER_DDIM, xs, y, cfg.cfg_scale, mt, levels, stream=stream)
    torch.cuda.synchronize()
    model.profile(False)
    sp = model.profile_read()["sampler"]
    lat = cfg.batch * cfg.in_channels * cfg.frames * cfg.height * cfg.width
    step_bytes = lat * 4 * 3          # read x and the eps channels, write x
    k_us = sp[0] / max(sp[1], 1) * 1e3
    sampler_line = {"kind": "DDIM (deterministic), levels 0.05..0.95", "steps": n_s,
                    "ms_per_step": s_ms / reps / n_s, "images_per_s": cfg.batch * n_s * reps / (s_ms / 1e3),
                    "update_kernel_us": k_us, "update_kernel_bytes": step_bytes,
                    "update_kernel_gbs": step_bytes / (k_us * 1e-6) / 1e9,
                    "launch": "CUDA graph replay of the whole loop" if not args.no_graph else "direct launches"}

    per, step_flops = kernel_flops(cfg)
    tokens = cfg.rows * cfg.tokens
    value = aggregate_rate(tokens, world, args.steps, total_ms / 1e3)
    ms_per_step = total_ms / args.steps
    pk, pk_kind = peaks()
    burst = pk["bf16_tflops"]
    sustained = pk.get("bf16_tflops_sustained", burst)
    achieved_tf = step_flops / (ms_per_step / 1e3) / 1e12
    for k, v in kernels.items():
        if (per.get(k) or 0) > 0 and v["us_per_launch"] > 0:
            v["tflops"] = per[k] / (v["us_per_launch"] * 1e-6) / 1e12
            v["frac_of_burst_bf16"] = v["tflops"] / burst
    if "ln" in kernels and kernels["ln"]["us_per_launch"] > 0:
        kernels["ln"]["gbs"] = ln_bytes(cfg) / (kernels["ln"]["us_per_launch"] * 1e-6) / 1e9
        kernels["ln"]["frac_of_hbm"] = kernels["ln"]["gbs"] / pk["hbm_gbs"]

    # the roofline of the kernel kind with the largest in-pipeline time per step
    top = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    avg_s = kernels[top]["us_per_launch"] * 1e-6
    traffic = TRAFFIC_BYTES.get(top)
    if (per.get(top) or 0) > 0:
        ach = per[top] / avg_s / 1e12
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": burst, "unit": "TFLOP/s",
                "frac": ach / burst, "traffic": traffic,
                "peak_source": f"{pk_kind} bf16 dense, burst (cuBLAS 8192^3, best of 10)",
                "frac_of_sustained": ach / sustained, "frac_of_nominal": ach / NOMINAL_BF16_TFLOPS,
                "avg_launch_us": avg_s * 1e6, "flops_per_launch": per[top],
                "timing": "CUDA events around each launch of this kind (others overlapped as usual)"}
    else:
        ach = ln_bytes(cfg) / avg_s / 1e9
        roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "traffic": traffic, "peak_source": f"{pk_kind} copy bandwidth",
                "avg_launch_us": avg_s * 1e6, "bytes_per_launch": ln_bytes(cfg),
                "timing": "CUDA events around each launch of this kind (others overlapped as usual)"}
    if traffic is not None:
        roof["traffic_source"] = TRAFFIC_SOURCE
    sm_mhz = clocks.get("sm_mhz")

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "ms_per_step_median": ms_median,
        "ms_per_step_min": ms_min, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) latents, N(0,0.02) weights)",
        "config": {"workload": workload_desc(cfg), "global_batch": cfg.batch * world, "rows_per_gpu": cfg.rows,
                   "tokens_per_step_per_gpu": tokens, "seq_len": cfg.tokens,
                   "l2": "flushed between timed steps (256 MB write outside the events)",
                   "parallelism": f"replicas x{world} (weak scaling, no data-path collective)",
                   "launch": "direct launches" if args.no_graph else "CUDA graph replay of the whole forward"},
        "images_per_s": cfg.batch * world * args.steps / (total_ms / 1e3),
        "pct_of_bf16_peak": {"achieved_tflops": achieved_tf, "peak_tflops": burst, "frac": achieved_tf / burst,
                             "peak_source": f"{pk_kind} burst (cuBLAS bf16 8192^3)",
                             "frac_of_sustained": achieved_tf / sustained, "sustained_tflops": sustained,
                             "frac_of_nominal_2250": achieved_tf / NOMINAL_BF16_TFLOPS,
                             "sm_mhz_median": sm_mhz,
                             "ms_x_mhz_per_step": ms_per_step * sm_mhz if sm_mhz else None},
        "roofline": roof,
        "kernels": kernels,
        "kernels_sum_ms": sum(v["ms_per_step"] for v in kernels.values()),
        "kernels_marginal_sum_ms": sum(v.get("marginal_us_per_launch", 0.0) * v["launches_per_step"] / 1e3
                                       for v in kernels.values()),
        "e2e": {"value": aggregate_rate(tokens, world, args.steps, e2e_s), "unit": "tokens/s",
                "h2d_bytes_per_step": int(xh.numel() * 4 + th.numel() * 4 + yh.numel() * 4),
                "d2h_bytes_per_step": int(oh.numel() * 4), "api": "dit_forward_host"},
        "gpu_launches": model.launch_count(cfg.batch, cfg.cfg_scale) * args.steps,
        "sampler": sampler_line,
        "clocks": clocks,
        "device_status": status,
    }
    if rank == 0 and world == 1:
        line["gemm_vs_cublas"] = gemm_reference(cfg, kernels, flush)
        line["gemm_vs_cublas_note"] = ("cuBLAS writes plain bf16; the library's kernels fuse bias + GELU, the gated "
                                       "residual reduce-add into the float32 stream and the head-major Q/K/V^T scatter")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, weights)
    del weights
    if args.all_configs and world == 1:
        model.close()
        line["all_configs"] = all_configs(min(args.steps, 30), max(args.warmup, 3), not args.no_graph, flush, burst)
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
