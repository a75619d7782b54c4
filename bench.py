#!/usr/bin/env python
"""Benchmark of the Wan 2.1 DiT forward hot path on B200.

One step = one ``wan_dit_stack_fwd`` call with one block on the 1.3B block shape at
480P, 81 frames (latent 16x21x60x104 -> 32760 tokens, dim 1536, 12 heads, FFN 8960,
512 text tokens): (1,2,2) patchify, the shared timestep MLP, one DiT block
(modulated LN, self-attention, cross-attention, gated FFN) and the head. Weights and
inputs are seeded synthetic data (N(0,0.02) weights, N(0,1) latents and context).

Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle instead.
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on the data
path; value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DiT block fwd tokens/sec and attention/GEMM TFLOP/s (% of B200 bf16 peak)"
UNIT = "tokens/s"
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan13b_480p_block")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def block_flops(w) -> float:
    """Algorithmic FLOPs of one block (2 per multiply-add)."""
    L, D, F, Lc, Li = w.tokens, w.dim, w.ffn, w.text_len, w.img_len
    f = 2 * L * D * 3 * D + 4 * L * L * D + 2 * L * D * D          # QKV, self-attention, O
    f += 2 * L * D * D + 4 * Lc * D * D + 4 * L * Lc * D + 2 * L * D * D  # cross q, kv, attention, o
    if Li:
        f += 4 * Li * D * D + 4 * L * Li * D + 2 * L * D * D       # image kv, attention, wider o
    f += 4 * L * D * F                                              # FFN
    return float(f) * w.batch


def step_flops(w) -> float:
    patch = 2.0 * w.tokens * w.in_ch * 4 * w.dim * w.batch
    head = 2.0 * w.tokens * w.dim * w.out_ch * 4 * w.batch
    tmlp = 2.0 * (w.freq_dim * w.dim + 6 * w.dim * w.dim) * w.batch
    return patch + tmlp + w.n_blocks * block_flops(w) + head


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def attn_traffic_per_launch():
    """DRAM bytes (read + write) per self-attention launch from the committed ncu
    summary, or None when the kernel source changed since the counters were taken."""
    p = os.path.join(PROFILES, "attn_fwd_tc_kernel__self_L32760_H12.md")
    src = os.path.join(ROOT, "video_diffusion_transformer_wan_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(p):
        return None
    sha = byts = None
    for line in open(p):
        if line.startswith("- attn_tc.cu sha256:"):
            sha = line.split(":", 1)[1].strip()
        elif line.startswith("- dram bytes per launch (read+write):"):
            byts = float(line.split(":", 1)[1])
    if sha != hashlib.sha256(open(src, "rb").read()).hexdigest():
        return None
    return byts


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else (os.cpu_count() or 1)
    except Exception:
        return os.cpu_count() or 1


def max_over_ranks(v: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the slowest replica sets the time)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, tokens_per_step: float, ms_per_step: float) -> float:
    """Whole-job tokens/s of `world` independent replicas timed by the slowest one."""
    return world * tokens_per_step / (ms_per_step / 1e3)


def _oracle_prefix(inp):
    from oracle import wan_oracle as O
    x = O.patchify(inp["noise"][0], inp["w_p"], inp["b_p"])
    e = O.time_mlp(float(inp["t"][0]), inp["w_t1"], inp["b_t1"], inp["w_t2"], inp["b_t2"])
    return x, e


def _oracle_rows(w, inp, x, e, S, seed=1) -> float:
    """Seconds the oracle takes for the block on S sampled query rows (keys and values
    over all rows, since self-attention needs them)."""
    from oracle import wan_oracle as O
    from wan_inputs import sample_rows
    rows = sample_rows(w.tokens, count=S, seed=seed)
    t0 = time.perf_counter()
    O.dit_block(x, e, inp["blocks"][0], inp["ctx"][0], w.heads, rows=rows)
    return time.perf_counter() - t0


def oracle_calibrate(w, inp, s_small=128, s_big=512):
    """Time the CPU oracle on a bounded sample of one step: patchify and the timestep MLP
    on all tokens, then the block for two query-row sample sizes. Returns
    (t_prefix, fixed, per_row, seconds_spent): the full block is fixed + per_row * L."""
    t0 = time.perf_counter()
    x, e = _oracle_prefix(inp)
    t_pre = time.perf_counter() - t0
    ta = _oracle_rows(w, inp, x, e, s_small)
    tb = _oracle_rows(w, inp, x, e, s_big)
    per_row = max((tb - ta) / (s_big - s_small), 1e-9)
    fixed = max(ta - per_row * s_small, 0.0)
    return t_pre, fixed, per_row, time.perf_counter() - t0, (x, e)


def oracle_sample(w, inp, s_small=128, s_big=512):
    t_pre, fixed, per_row, spent, _ = oracle_calibrate(w, inp, s_small, s_big)
    t_full = t_pre + fixed + per_row * w.tokens
    desc = (f"fp64 numpy oracle: patchify + timestep MLP on all {w.tokens} tokens, then the block for "
            f"{s_small} and {s_big} sampled query rows (K/V over all rows each time); the full-block time is "
            f"extrapolated linearly in query rows: {t_full:.1f} s per step")
    return w.tokens * w.batch / t_full, spent, desc


def run_reference(args, w):
    """The oracle arm. Warm-up calibrates the per-row cost of the oracle; each timed step
    evaluates the block on one bounded sample of query rows (keys and values over all
    rows) and extrapolates its measured time to all L rows with that per-row cost."""
    from wan_inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = make_inputs(w, seed=0, n_blocks=1, block_input=False)
    t_pre, fixed, per_row, _, (x, e) = oracle_calibrate(w, inp, 64, 256)
    for _ in range(max(args.warmup - 1, 0)):
        _oracle_rows(w, inp, x, e, 64)
    S = 64
    vals = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        x, e = _oracle_prefix(inp)
        ts = time.perf_counter() - t0 + _oracle_rows(w, inp, x, e, S, seed=100 + i)
        vals.append(w.tokens * w.batch / (ts + per_row * (w.tokens - S)))
    value = statistics.median(vals)
    cores = blas_threads()
    desc = (f"fp64 numpy oracle per step: patchify + timestep MLP on all tokens and the block for {S} sampled "
            f"query rows (K/V over all rows); the remaining rows are added at the per-row cost calibrated in "
            f"warm-up ({per_row * 1e3:.2f} ms/row)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * w.tokens * w.batch / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "tokens": w.tokens, "dim": w.dim, "heads": w.heads,
                   "ffn": w.ffn, "text_tokens": w.text_len, "blocks": 1, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from wan_inputs import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import video_diffusion_transformer_wan_b200 as wan
    from video_diffusion_transformer_wan_b200.model import DitModel, config_for, to_device

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    # Independent replicas: every rank draws its own sample (seed = rank).
    inp = make_inputs(w, seed=rank, block_input=False)
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    act = model.act
    B, F, H, W, L = w.batch, w.frames, w.height, w.width, w.tokens
    if w.flow_matching:
        t_host = (1000.0 * inp["u"]).astype("float32")
    else:
        t_host = inp["t"]
    noise = inp["noise"]
    img_ctx = None
    lat_host_np = noise
    if w.i2v:
        lat_host_np = None
    lat = to_device(noise, act)
    if w.i2v:
        import numpy as np
        cond = to_device(inp["cond"], act)
        keep = np.zeros((B, 1 + 4 * (F - 1)), np.uint8)
        keep[:, 0] = 1
        lat36 = torch.empty(B, 36, F, H, W, dtype=act, device="cuda")
        wan.i2v_input(cfg, lat, cond, torch.from_numpy(keep).cuda(), lat36)
        lat = lat36
        feat = to_device(inp["img_feat"], act)
        img_ctx = torch.empty(B, w.img_len, w.dim, dtype=act, device="cuda")
        iws = torch.empty(2 * B * w.img_len * w.dim * 2, dtype=torch.uint8, device="cuda")
        wan.image_context_fwd(cfg, feat, model.image_table, img_ctx, iws)
    t = torch.from_numpy(t_host).cuda()
    ctx = to_device(inp["ctx"], act)
    v = torch.empty(B, w.out_ch, F, H, W, dtype=torch.float32, device="cuda")
    ws = torch.empty(wan.workspace_bytes(cfg, B, L, w.text_len, w.img_len), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        wan.dit_stack_fwd(cfg, lat, t, model.stack_table, model.block_tables, ctx, img_ctx, v, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = wan.device_status()
    if status != 0:
        raise RuntimeError(f"device status {wan.status_string(status)} after warm-up")

    # ---------------- device-resident timed region (inputs already in HBM)
    sampler = ClockSampler(local)
    wan.trace_reset()
    wan.trace_enable(True)
    launches0 = wan.launch_count()
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.1)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    launches = wan.launch_count() - launches0
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    recs = wan.trace_launches()
    wan.trace_enable(False)
    ms_step = ms_total / args.steps
    tokens_step = B * L
    value = replica_throughput(world, tokens_step, ms_step)
    flops = step_flops(w)

    # dominant kernel: the self-attention launch (largest attention work per step)
    attn = [(ms, work) for k, ms, work in recs if k == wan.KIND_ATTN]
    top = max(wk for _, wk in attn)
    self_attn = [(ms, wk) for ms, wk in attn if wk == top]
    attn_ms = statistics.mean(ms for ms, _ in self_attn)
    peaks, peak_src = load_peaks()
    achieved = top / (attn_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    kind_ms = {}
    for k, ms, _ in recs:
        kind_ms[k] = kind_ms.get(k, 0.0) + ms
    gemm_work = sum(wk for k, _, wk in recs if k == wan.KIND_GEMM)
    norm = [(ms, wk) for k, ms, wk in recs if k == wan.KIND_NORM]

    # ---------------- end to end through the C ABI with host buffers
    # Every step copies its inputs from pinned host memory and its velocity back. Two
    # sets of device buffers and an upload and a download stream let step k+1's inputs
    # and step k-1's result cross PCIe while step k computes; the timed interval covers
    # the first upload to the last download.
    lat_h = torch.empty(lat.shape, dtype=act, pin_memory=True)
    lat_h.copy_(lat.cpu())
    t_h = torch.from_numpy(t_host).pin_memory()
    ctx_h = torch.empty(ctx.shape, dtype=act, pin_memory=True)
    ctx_h.copy_(ctx.cpu())
    v_h = torch.empty(v.shape, dtype=torch.float32, pin_memory=True)
    h2d = lat_h.numel() * lat_h.element_size() + t_h.numel() * 4 + ctx_h.numel() * ctx_h.element_size()
    d2h = v_h.numel() * 4
    bufs = [(lat, t, ctx, v), (torch.empty_like(lat), torch.empty_like(t), torch.empty_like(ctx), torch.empty_like(v))]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in range(2)]      # inputs of the buffer set uploaded
    done = [torch.cuda.Event() for _ in range(2)]       # step on the buffer set finished
    drained = [torch.cuda.Event() for _ in range(2)]    # its velocity downloaded

    def e2e_run(n):
        for k in range(n):
            i = k % 2
            lat_i, t_i, ctx_i, v_i = bufs[i]
            with torch.cuda.stream(up):
                if k >= 2:
                    up.wait_event(drained[i])
                lat_i.copy_(lat_h, non_blocking=True)
                t_i.copy_(t_h, non_blocking=True)
                ctx_i.copy_(ctx_h, non_blocking=True)
                ready[i].record(up)
            stream.wait_event(ready[i])
            wan.dit_stack_fwd(cfg, lat_i, t_i, model.stack_table, model.block_tables, ctx_i, img_ctx, v_i, ws)
            done[i].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(done[i])
                v_h.copy_(v_i, non_blocking=True)
                drained[i].record(down)

    e2e_run(2)
    barrier()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    up.wait_event(e2)
    down.wait_event(e2)
    e2e_run(args.steps)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e2.elapsed_time(e3), world, "cuda") / args.steps
    e2e_value = replica_throughput(world, tokens_step, e2e_ms)
    status = wan.device_status()
    if status != 0:
        raise RuntimeError(f"device status {wan.status_string(status)} after timing")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, spent, desc = oracle_sample(w, inp)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": desc,
               "seconds": round(spent, 1)}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) latents/context; random init, no checkpoint)",
            "config": {"workload": w.name,
                       "step": "wan_dit_stack_fwd: patchify + timestep MLP + %d block(s) + head" % w.n_blocks,
                       "batch": B, "latent": [w.in_ch, F, H, W], "tokens": L, "dim": w.dim, "heads": w.heads,
                       "ffn": w.ffn, "text_tokens": w.text_len, "image_tokens": w.img_len,
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": "inputs larger than L2 (per-step working set > 1 GB of activations)"},
            "tflops": flops / (ms_step / 1e3) / 1e12 * world,
            "pct_bf16_peak": flops / (ms_step / 1e3) / 1e12 / peak,
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_tc_kernel (self-attention)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "work_per_launch": top, "ms_per_launch": attn_ms,
                         "traffic": attn_traffic_per_launch()},
            "kernels_ms_per_step": {
                "attention": kind_ms.get(wan.KIND_ATTN, 0.0) / args.steps,
                "gemm": kind_ms.get(wan.KIND_GEMM, 0.0) / args.steps,
                "layernorm": kind_ms.get(wan.KIND_NORM, 0.0) / args.steps,
                "small": kind_ms.get(wan.KIND_SMALL, 0.0) / args.steps},
            "gemm_tflops": gemm_work / (kind_ms.get(wan.KIND_GEMM, 1e-9) / 1e3) / 1e12,
            "layernorm_gbs": (sum(wk for _, wk in norm) / (sum(ms for ms, _ in norm) / 1e3) / 1e9) if norm else None,
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
