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


def code_sha256(path):
    """sha256 of a CUDA source with its // comments, surrounding whitespace and blank
    lines removed: it changes with the code, not with the comments."""
    lines = []
    for line in open(path, encoding="utf-8"):
        code = line.split("//", 1)[0].strip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def attn_traffic_per_launch(w):
    """DRAM bytes (read + write) per self-attention launch from the committed ncu
    summary, or None when the kernel code changed since the counters were taken or
    the summary's launch shape (batch, tokens, heads) is not this workload's."""
    p = os.path.join(PROFILES, "attn_fwd_tc_kernel__self_L32760_H12.md")
    src = os.path.join(ROOT, "video_diffusion_transformer_wan_b200", "csrc", "attn_tc.cu")
    if not os.path.exists(p):
        return None
    sha = byts = shape = None
    for line in open(p):
        if line.startswith("- attn_tc.cu code sha256:"):
            sha = line.split(":", 1)[1].strip()
        elif line.startswith("- dram bytes per launch (read+write):"):
            byts = float(line.split(":", 1)[1])
        elif line.startswith("- launch shape (batch, tokens, heads):"):
            shape = tuple(int(v) for v in line.split(":", 1)[1].split(","))
    if sha != code_sha256(src):
        return None
    if shape != (w.batch, w.tokens, w.heads):
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


def _oracle_inputs(w, inp):
    """The oracle's view of one step's inputs: the latent (I2V: the 36-channel fusion),
    the timestep, the text context and the image context (computed outside the timed
    region, as the GPU step takes it precomputed)."""
    from oracle import wan_oracle as O
    lat = inp["noise"][0]
    img = None
    if w.i2v:
        keep = [1] + [0] * (4 * (w.frames - 1))
        lat = O.i2v_input(inp["noise"][0], inp["cond"][0], O.i2v_mask(keep, w.frames, w.height, w.width))
        img = O.image_context_mlp(inp["img_feat"][0], *(inp[k] for k in ["w_i1", "b_i1", "w_i2", "b_i2",
                                                                         "w_i3", "b_i3"]))
    t = float(1000.0 * inp["u"][0]) if w.flow_matching else float(inp["t"][0])
    return lat, t, inp["ctx"][0], img


def oracle_step_seconds(w, inp) -> float:
    """Seconds the fp64 oracle takes for exactly the work of one GPU step: ``dit_stack``
    with the workload's blocks (patchify, timestep MLP, every block on all tokens, head,
    unpatchify), one sample."""
    from oracle import wan_oracle as O
    lat, t, ctx, img = _oracle_inputs(w, inp)
    t0 = time.perf_counter()
    O.dit_stack(lat, t, inp, inp["blocks"], ctx, w.heads, img_ctx=img)
    return time.perf_counter() - t0


def oracle_row_model(w, inp, s_small=64, s_big=256):
    """Cross-check only (also the CPU warm-up): the block on two sampled query-row counts
    (keys and values over all rows), fitted as fixed + per_row * rows and extended to all
    L rows. Returns (model seconds per step, seconds spent)."""
    from oracle import wan_oracle as O
    from wan_inputs import sample_rows
    lat, t, ctx, img = _oracle_inputs(w, inp)
    t0 = time.perf_counter()
    x = O.patchify(lat, inp["w_p"], inp["b_p"])
    e = O.time_mlp(t, inp["w_t1"], inp["b_t1"], inp["w_t2"], inp["b_t2"])
    t_pre = time.perf_counter() - t0
    ts = []
    for S in (s_small, s_big):
        rows = sample_rows(w.tokens, count=S, seed=1)
        t1 = time.perf_counter()
        for blk in inp["blocks"]:
            O.dit_block(x, e, blk, ctx, w.heads, img_ctx=img, rows=rows)
        ts.append(time.perf_counter() - t1)
    per_row = max((ts[1] - ts[0]) / (s_big - s_small), 0.0)
    fixed = max(ts[0] - per_row * s_small, 0.0)
    return t_pre + fixed + per_row * w.tokens, time.perf_counter() - t0


def oracle_measure(w, inp):
    """The CPU baseline: warm-up and per-row cross-check, then the oracle timed over one
    whole step of the workload. Returns (tokens/s, step seconds, description, model seconds)."""
    model_s, _ = oracle_row_model(w, inp)
    step_s = oracle_step_seconds(w, inp)
    desc = (f"fp64 numpy oracle timed over one whole step of {w.name} ({w.n_blocks} block(s) on all "
            f"{w.tokens} tokens, patchify, timestep MLP and head): {step_s:.1f} s; warm-up: the block on 64 and "
            f"256 sampled query rows, whose linear per-row model predicts {model_s:.1f} s (cross-check only)")
    return w.tokens * w.batch / step_s, step_s, desc, model_s


def run_reference(args, w):
    """The oracle arm. The fp64 oracle is the slow program on the host cores; one of its
    steps at the 1.3B 480P shape takes on the order of 100 s, so the arm times ONE whole
    step (the same work as one GPU step) after a bounded warm-up, and says so: its
    ``steps`` is 1 whatever ``--steps`` asks for."""
    from wan_inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = make_inputs(w, seed=0, block_input=False)
    value, step_s, desc, model_s = oracle_measure(w, inp)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": 1, "steps_requested": args.steps, "warmup": 1, "warmup_requested": args.warmup,
        "ms_per_step": 1000.0 * step_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "tokens": w.tokens, "dim": w.dim, "heads": w.heads,
                   "ffn": w.ffn, "text_tokens": w.text_len, "image_tokens": w.img_len, "blocks": w.n_blocks,
                   "parallelism": "replicas"},
        "note": "one whole oracle step timed (about 100 s at this shape); the requested step count is not run",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                         "model_seconds": round(model_s, 1)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def choose_peak(peaks, peak_src, region_s):
    """The bf16 denominator for kernels timed inside a region of ``region_s`` seconds:
    the burst figure for a region under 1 s (the GPU does not reach its power-capped
    steady state in that time), the sustained one otherwise."""
    burst = region_s < 1.0
    key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    return {"value": peaks[key], "hbm_gbs": peaks["hbm_gbs"],
            "source": f"{peak_src} {key} ({'burst' if burst else 'sustained'}: timed region {region_s:.2f} s)"}


def kernel_report(w, recs, steps, ms_step, clocks):
    """Per-kernel durations and roofline fractions from the per-launch trace of ``steps``
    steps. In each step the first GEMM is the patchify projection and the last the head
    (both HBM-bound; algorithmic bytes = operands read once + output written once); the
    attention launch with the most work is the self-attention, the others are
    cross-attention; LayerNorm work is its algorithmic bytes."""
    import video_diffusion_transformer_wan_b200 as wan
    peaks, peak_src = load_peaks()
    peak = choose_peak(peaks, peak_src, ms_step * steps / 1e3)
    n = len(recs)
    per = n // steps if steps and n % steps == 0 else None
    if not per:
        raise RuntimeError(f"trace holds {n} launches, not a multiple of {steps} steps")
    B, L, D = w.batch, w.tokens, w.dim
    K = w.in_ch * 4
    patch_bytes = B * L * K * 2 + D * K * 2 + D * 2 + B * L * D * 4
    head_bytes = B * L * D * 2 + w.out_ch * 4 * D * 2 + w.out_ch * 4 * 2 + B * L * w.out_ch * 4 * 4
    acc = {k: [0.0, 0.0] for k in ["self_attention", "cross_attention", "gemm", "patchify_gemm", "head_gemm",
                                   "layernorm", "small"]}
    top = max(wk for k, _, wk in recs if k == wan.KIND_ATTN)
    # self-attention launches per step (one per block)
    n_sa = sum(1 for k, _, wk in recs[:per] if k == wan.KIND_ATTN and wk == top)
    for i in range(steps):
        chunk = recs[i * per:(i + 1) * per]
        gi = [j for j, (k, _, _) in enumerate(chunk) if k == wan.KIND_GEMM]
        for j, (k, ms, wk) in enumerate(chunk):
            if k == wan.KIND_ATTN:
                name = "self_attention" if wk == top else "cross_attention"
            elif k == wan.KIND_GEMM:
                name = "patchify_gemm" if j == gi[0] else "head_gemm" if j == gi[-1] else "gemm"
                if name != "gemm":
                    wk = patch_bytes if name == "patchify_gemm" else head_bytes
            elif k == wan.KIND_NORM:
                name = "layernorm"
            else:
                name = "small"
            acc[name][0] += ms
            acc[name][1] += wk
    mhz = clocks.get("sm_mhz")
    out = {}
    for name, (ms, wk) in acc.items():
        d = {"ms_per_step": ms / steps}
        if name in ("self_attention", "cross_attention", "gemm") and ms > 0:
            d.update({"tflops": wk / (ms / 1e3) / 1e12, "bound": "tensor"})
            d["frac"] = d["tflops"] / peak["value"]
        elif name in ("patchify_gemm", "head_gemm", "layernorm") and ms > 0:
            d.update({"gbs": wk / (ms / 1e3) / 1e9, "bound": "hbm"})
            d["frac"] = d["gbs"] / peak["hbm_gbs"]
        d["sm_mhz"] = mhz
        out[name] = d
    out["peaks"] = {"bf16_tflops": peak["value"], "bf16_source": peak["source"], "hbm_gbs": peak["hbm_gbs"],
                    "hbm_source": f"{peak_src} hbm_gbs"}
    sa_ms = acc["self_attention"][0] / (steps * n_sa)
    roofline = {"bound": "tensor", "kernel": "attn_fwd_tc_kernel (self-attention)",
                "achieved": top / (sa_ms / 1e3) / 1e12, "peak": peak["value"], "unit": "TFLOP/s",
                "frac": top / (sa_ms / 1e3) / 1e12 / peak["value"], "peak_source": peak["source"],
                "sm_mhz": mhz, "work_per_launch": top, "ms_per_launch": sa_ms,
                "traffic": attn_traffic_per_launch(w)}
    return out, roofline, peak


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

    # ---------------- device-resident timed region (inputs already in HBM), untraced
    sampler = ClockSampler(local)
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
    ms_step = ms_total / args.steps
    tokens_step = B * L
    value = replica_throughput(world, tokens_step, ms_step)
    flops = step_flops(w)

    # ---------------- the same K steps again with the per-launch trace (CUDA events
    # around every launch on the launch stream): per-kernel durations
    sampler_t = ClockSampler(local)
    wan.trace_reset()
    wan.trace_enable(True)
    barrier()
    torch.cuda.synchronize()
    sampler_t.start()
    time.sleep(0.1)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    for _ in range(args.steps):
        step()
    e5.record(stream)
    torch.cuda.synchronize()
    clocks_traced = sampler_t.stop()
    barrier()
    traced_ms_step = e4.elapsed_time(e5) / args.steps
    recs = wan.trace_launches()
    wan.trace_enable(False)
    kernels, roofline, peak = kernel_report(w, recs, args.steps, traced_ms_step, clocks_traced)

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
        v_cpu, step_s, desc, model_s = oracle_measure(w, inp)
        cpu = {"value": v_cpu, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": desc,
               "seconds": round(step_s, 1), "model_seconds": round(model_s, 1)}

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
            "pct_bf16_peak": flops / (ms_step / 1e3) / 1e12 / peak["value"],
            "pct_bf16_peak_basis": peak["source"],
            "roofline": roofline,
            "kernels": kernels,
            "traced_ms_per_step": traced_ms_step,
            "hbm_peak_gbs": peak["hbm_gbs"],
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": clocks,
            "clocks_traced": clocks_traced,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
