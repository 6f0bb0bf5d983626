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
import math
import os
import statistics
import subprocess
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
# DRAM bytes (read + write) of one launch of each kernel, from the cold-cache ncu captures
# summarised in profiles/xl2_cfg256_kernels_ncu.md; set to None when a kernel changes.
TRAFFIC_BYTES = {"fc1": 58.6e6, "fc2": 128.5e6, "qkv": 43.0e6, "proj": 59.5e6, "attn": 65.4e6, "ln": 38.1e6}
# fallback peaks (used only when MEASURED_PEAKS.json is absent)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


def workload_desc(cfg):
    return (f"DiT-XL/2 CFG 256px: {cfg.batch} latents {cfg.in_channels}x{cfg.height}x{cfg.width} -> "
            f"{cfg.rows} rows x {cfg.tokens} tokens, d={cfg.hidden}, {cfg.depth} blocks, {cfg.heads} heads, "
            f"s={cfg.cfg_scale}")


def kernel_flops(cfg):
    """Algorithmic FLOPs (2 per multiply-add) per launch of each kernel kind, and per step."""
    R, T, d, mlp, H = cfg.rows, cfg.tokens, cfg.hidden, cfg.mlp_hidden, cfg.heads
    dh = cfg.head_dim
    M = R * T
    nmod = (6 * cfg.depth + 2) * d
    per = {
        "cond": 2 * R * (cfg.freq_dim * d + d * d),
        "adaln": 2 * R * nmod * d,
        "patch": 2 * M * d * cfg.patch_dim,
        "qkv": 2 * M * 3 * d * d,
        "attn": 4 * R * H * T * T * dh,
        "proj": 2 * M * d * d,
        "fc1": 2 * M * mlp * d,
        "fc2": 2 * M * d * mlp,
        "decode": 2 * M * d * cfg.out_dim,
        "ln": 0,
    }
    step = (per["cond"] + per["adaln"] + per["patch"] + per["decode"] +
            cfg.depth * (per["qkv"] + per["attn"] + per["proj"] + per["fc1"] + per["fc2"]))
    return per, step


def ln_bytes(cfg):
    M = cfg.rows * cfg.tokens
    return M * cfg.hidden * (4 + 2)  # read f32 residual, write bf16


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str | None):
        self.rows = []
        self.proc = None
        self.dev = device_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.dev:
            cmd += ["-i", self.dev]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")

        sm = [num(r[1]) for r in self.rows]
        mx = [num(r[2]) for r in self.rows]
        pw = [num(r[3]) for r in self.rows]
        loaded = [s for s, p in zip(sm, pw) if p > 200] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            for name, flag in zip(names, r[5:9]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(self.rows), "power_w_max": max(pw)}


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


def time_config(cfg, steps, warmup, graph, flush):
    """Device time of `steps` whole forwards of `cfg` (seeded weights and inputs, L2 flushed between
    steps outside the events).  Returns per-step milliseconds."""
    import torch
    from diffusion_transformer_denoiser_dit_b200 import DiT
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_OPT_USE_GRAPH
    model = DiT(cfg, S.make_weights(cfg))
    model.set_option(DIT_OPT_USE_GRAPH, 1 if graph else 0)
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


def all_configs(steps, warmup, graph, flush, peak_tf):
    res = {}
    for name, cfg in (("c1 S/8 fp32", S.DIT_S8_F32), ("c2 B/4 bf16", S.DIT_B4_BF16),
                      ("c3 XL/2 CFG 256px", S.DIT_XL2_CFG256), ("c4 XL/2 CFG 512px", S.DIT_XL2_CFG512),
                      ("c5 video RF 4096 tokens", S.VIDEO_RF)):
        ms = time_config(cfg, steps, warmup, graph, flush)
        med = statistics.median(ms)
        _, fl = kernel_flops(cfg)
        tf = fl / (med / 1e3) / 1e12
        res[name] = {"ms_per_step_median": med, "ms_per_step_min": min(ms),
                     "tokens_per_s": cfg.rows * cfg.tokens / (med / 1e3),
                     "samples_per_s": cfg.batch / (med / 1e3), "tflops": tf,
                     "frac_of_sustained_bf16": tf / peak_tf if cfg.dtype == S.DTYPE_BF16 else None,
                     "dtype": "bf16" if cfg.dtype == S.DTYPE_BF16 else "f32",
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
    ap.add_argument("--all-configs", action="store_true",
                    help="also time the other workloads (S/8 fp32, B/4, XL/2 512px CFG, video) and report them under "
                         "'all_configs' in the same JSON line")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from diffusion_transformer_denoiser_dit_b200 import DiT
    from diffusion_transformer_denoiser_dit_b200.binding import DIT_OPT_USE_GRAPH

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    cfg = CFG
    weights = S.make_weights(cfg)
    model = DiT(cfg, weights)
    model.set_option(DIT_OPT_USE_GRAPH, 0 if args.no_graph else 1)
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

    dev_id = None
    try:
        dev_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(dev_id)
    sampler.start()
    time.sleep(0.3)
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

    # per-kernel durations: a second pass with events around every launch
    model.profile(True)
    for i in range(args.steps):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    model.profile(False)
    prof = model.profile_read()

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
    sustained = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    achieved_tf = step_flops / (ms_per_step / 1e3) / 1e12

    # dominant kernel by device time
    kinds = {k: v for k, v in prof.items() if v[1] > 0}
    top = max(kinds, key=lambda k: kinds[k][0])
    top_ms, top_n = kinds[top]
    avg_s = top_ms / top_n / 1e3
    if per.get(top, 0) > 0:
        ach = per[top] / avg_s / 1e12
        roof = {"kernel": top, "bound": "tensor", "achieved": ach, "peak": sustained, "unit": "TFLOP/s",
                "frac": ach / sustained, "traffic": TRAFFIC_BYTES.get(top),
                "peak_source": f"{pk_kind} bf16 dense, sustained (cuBLAS 8192^3 loop)",
                "avg_launch_us": avg_s * 1e6, "flops_per_launch": per[top]}
    else:
        ach = ln_bytes(cfg) / avg_s / 1e9
        roof = {"kernel": top, "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "traffic": TRAFFIC_BYTES.get(top), "peak_source": f"{pk_kind} copy bandwidth",
                "avg_launch_us": avg_s * 1e6}
    kernels = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps}
               for k, v in kinds.items()}
    for k in kernels:
        if per.get(k, 0) > 0 and kinds[k][1] > 0:
            kernels[k]["tflops"] = per[k] / (kinds[k][0] / kinds[k][1] / 1e3) / 1e12
    ln_k = kinds.get("ln")
    if ln_k:
        kernels["ln"]["gbs"] = ln_bytes(cfg) / (ln_k[0] / ln_k[1] / 1e3) / 1e9

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
        "pct_of_bf16_peak": {"achieved_tflops": achieved_tf, "peak_tflops": sustained,
                             "frac": achieved_tf / sustained, "peak_source": f"{pk_kind} sustained",
                             "frac_of_nominal_2250": achieved_tf / 2250.0},
        "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": aggregate_rate(tokens, world, args.steps, e2e_s), "unit": "tokens/s",
                "h2d_bytes_per_step": int(xh.numel() * 4 + th.numel() * 4 + yh.numel() * 4),
                "d2h_bytes_per_step": int(oh.numel() * 4), "api": "dit_forward_host"},
        "gpu_launches": model.launch_count(cfg.batch, cfg.cfg_scale) * args.steps,
        "sampler": sampler_line,
        "clocks": sampler.summary(),
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, weights)
    del weights
    if args.all_configs and world == 1:
        model.close()
        line["all_configs"] = all_configs(min(args.steps, 30), max(args.warmup, 3), not args.no_graph, flush, sustained)
    if rank == 0:
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
