"""Single-kernel micro-benchmark through the C ABI (CUDA-event timing), also the
command the committed ncu summaries were captured with.

  python -m video_diffusion_transformer_wan_b200.kernel_bench attention --L 32760 --heads 12
  python -m video_diffusion_transformer_wan_b200.kernel_bench gemm --M 32760 --N 4608 --K 1536 --epi store
  python -m video_diffusion_transformer_wan_b200.kernel_bench layernorm --L 32760 --dim 1536
  python -m video_diffusion_transformer_wan_b200.kernel_bench patchify --frames 21 --height 60 --width 104
  python -m video_diffusion_transformer_wan_b200.kernel_bench head --frames 21 --height 60 --width 104
  python -m video_diffusion_transformer_wan_b200.kernel_bench sample --blocks 30 --steps 2

Inputs are random device tensors (the kernels' timing does not depend on values); the
``sample`` mode draws the 1.3B 480P workload's seeded weights and times the guided
Euler loop (one call of ``steps`` steps, conditional and unconditional branches as one
batch of two).
Prints one JSON line with the per-launch time and the achieved rate.
"""
from __future__ import annotations

import argparse
import json

import torch

import video_diffusion_transformer_wan_b200 as wan


def _time(fn, iters: int, warmup: int) -> float:
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / max(iters, 1)


def _sample(a) -> dict:
    import dataclasses

    from wan_inputs import WORKLOADS, make_inputs

    from .model import DitModel, config_for, to_device
    w = dataclasses.replace(WORKLOADS["wan13b_480p_block"], n_blocks=a.blocks)
    inp = make_inputs(w, seed=0, block_input=False, uncond=True)
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    B, F, H, W, L, D = w.batch, w.frames, w.height, w.width, w.tokens, w.dim
    noise = to_device(inp["noise"], model.act)
    ctx, ctx_u = to_device(inp["ctx"], model.act), to_device(inp["ctx_uncond"], model.act)
    out = torch.empty(B, w.out_ch, F, H, W, dtype=torch.float32, device="cuda")
    cache = wan.DiffusionCache(*[int(v) for v in a.cache.split(",")]) if a.cache else None
    tables, scales = model.block_tables, None
    if a.fp8:
        from .model import Fp8Block
        fbs = [Fp8Block(cfg, b, attention_fp8=a.fp8_attention) for b in model.blocks]
        tables, scales = [f.table for f in fbs], [f.scale_table for f in fbs]
    ws = torch.empty(wan.sample_workspace_bytes(cfg, a.blocks, B, F, H, W, w.text_len, 0, cache, fp8=a.fp8),
                     dtype=torch.uint8, device="cuda")
    ms = _time(lambda: wan.sample_euler_cfg(cfg, noise, a.steps, a.guidance, model.stack_table, tables, ctx, ctx_u,
                                            None, out, ws, cache=cache, fp8_scales=scales), a.iters, a.warmup)
    Lc, Fd = w.text_len, w.ffn
    # per step; the text K|V projections are made once per call and not counted
    block = 2 * L * D * 3 * D + 4 * L * L * D + 3 * 2 * L * D * D + 4 * L * Lc * D + 4 * L * D * Fd
    flops_step = 2 * B * (a.blocks * block + 2 * L * D * 64 * 2)
    return dict(workload=w.name, blocks=a.blocks, euler_steps=a.steps, cache=a.cache or None, fp8=a.fp8,
                fp8_attention=a.fp8 and a.fp8_attention, ms_per_call=ms,
                ms_per_euler_step=ms / a.steps,
                latent_tokens_per_s=B * L * a.steps / (ms / 1e3),
                tflops_uncached_equivalent=flops_step * a.steps / ms / 1e9)


def _block(a) -> dict:
    """One DiT block call (bf16 or FP8 linear layers) on a workload's shapes."""
    from wan_inputs import WORKLOADS, make_inputs

    from .model import DitModel, Fp8Block, config_for, to_device
    w = WORKLOADS[a.workload]
    inp = make_inputs(w, seed=0, n_blocks=1)
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    x0 = to_device(inp["x"], torch.float32)
    e = to_device(inp["e"], torch.float32)
    ctx = to_device(inp["ctx"], model.act)
    x = x0.clone()
    B, L = w.batch, w.tokens
    if a.fp8:
        fb = Fp8Block(cfg, model.blocks[0], attention_fp8=a.fp8_attention)
        ws = torch.empty(wan.fp8_workspace_bytes(cfg, B, L, w.text_len), dtype=torch.uint8, device="cuda")
        ms = _time(lambda: wan.dit_block_fp8_fwd(cfg, x, e, ctx, None, fb.table, fb.scale_table, ws), a.iters,
                   a.warmup)
    else:
        ws = torch.empty(wan.workspace_bytes(cfg, B, L, w.text_len), dtype=torch.uint8, device="cuda")
        ms = _time(lambda: wan.dit_block_fwd(cfg, x, e, ctx, None, model.block_tables[0], ws), a.iters, a.warmup)
    D, F, Lc = w.dim, w.ffn, w.text_len
    flops = B * (2 * L * D * 3 * D + 4 * L * L * D + 3 * 2 * L * D * D + 4 * Lc * D * D + 4 * L * Lc * D
                 + 4 * L * D * F)
    return dict(workload=w.name, fp8=a.fp8, fp8_attention=a.fp8 and a.fp8_attention, ms=ms,
                tokens_per_s=B * L / (ms / 1e3), tflops=flops / ms / 1e9)


def _patch_or_head(a, g) -> dict:
    """wan_patchify (patch gather + the K = in_ch*4 projection, fp32 store) or wan_head_fwd
    (plain LN + the N = 64 projection scattered into the latent) on one 480P-sized latent.
    Both projections are HBM-bound; algorithmic bytes: inputs read once, outputs written
    once (patchify: latent, gathered patches written and read, W, x; head: x, the LN
    output written and read, W, v)."""
    D, F, H, W = a.dim, a.frames, a.height, a.width
    L = F * (H // 2) * (W // 2)
    cfg = wan.make_config(D, D // 128, 4 * D, in_ch=a.in_ch)
    if a.kernel == "patchify":
        K = a.in_ch * 4
        lat = torch.randn(1, a.in_ch, F, H, W, device="cuda", generator=g).to(torch.bfloat16)
        wp = (torch.randn(D, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        bp = torch.zeros(D, dtype=torch.bfloat16, device="cuda")
        x = torch.empty(1, L, D, dtype=torch.float32, device="cuda")
        ws = torch.empty(L * K * 2, dtype=torch.uint8, device="cuda")
        ms = _time(lambda: wan.patchify(cfg, lat, wp, bp, x, ws), a.iters, a.warmup)
        byts = L * K * 2 * 3 + D * K * 2 + L * D * 4.0
    else:
        x = torch.randn(1, L, D, device="cuda", generator=g)
        wh = (torch.randn(64, D, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        bh = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
        v = torch.empty(1, 16, F, H, W, dtype=torch.float32, device="cuda")
        ws = torch.empty(L * D * 2, dtype=torch.uint8, device="cuda")
        ms = _time(lambda: wan.head_fwd(cfg, x, F, H, W, wh, bh, v, ws), a.iters, a.warmup)
        byts = L * D * 4 + L * D * 2 * 2 + 64 * D * 2 + L * 64 * 4.0
    return dict(L=L, dim=D, ms=ms, gbs=byts / ms / 1e6, alg_bytes=byts)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["attention", "gemm", "layernorm", "sample", "block", "patchify", "head"])
    ap.add_argument("--fp8", action="store_true", help="attention / gemm / block / sample: E4M3 operands (kind::f8f6f4)")
    ap.add_argument("--fp8-attention", action="store_true",
                    help="block / sample with --fp8: the self-attention on E4M3 operands as well")
    ap.add_argument("--no-split", action="store_true",
                    help="attention: no workspace, so a partial last wave is not split over the keys")
    ap.add_argument("--workload", default="wan13b_480p_block", help="block: workload name")
    ap.add_argument("--blocks", type=int, default=30, help="sample: DiT blocks")
    ap.add_argument("--steps", type=int, default=2, help="sample: Euler steps per call")
    ap.add_argument("--guidance", type=float, default=5.0)
    ap.add_argument("--cache", default="", help="sample: diffusion cache attn_start,attn_interval,cfg_start,cfg_interval")
    ap.add_argument("--L", type=int, default=32760)
    ap.add_argument("--Lk", type=int, default=0, help="key length (default: L, self-attention)")
    ap.add_argument("--heads", type=int, default=12)
    ap.add_argument("--dim", type=int, default=1536)
    ap.add_argument("--M", type=int, default=32760)
    ap.add_argument("--N", type=int, default=4608)
    ap.add_argument("--K", type=int, default=1536)
    ap.add_argument("--epi", choices=["store", "gelu", "residual", "f32"], default="store")
    ap.add_argument("--frames", type=int, default=21, help="patchify / head: latent frames")
    ap.add_argument("--height", type=int, default=60, help="patchify / head: latent height")
    ap.add_argument("--width", type=int, default=104, help="patchify / head: latent width")
    ap.add_argument("--in-ch", type=int, default=16, help="patchify: latent channels")
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=2)
    a = ap.parse_args(argv)
    g = torch.Generator(device="cuda").manual_seed(0)
    out = {"kernel": a.kernel}
    if a.kernel == "attention":
        D = a.heads * 128
        Lk = a.Lk or a.L
        cfg = wan.make_config(D, a.heads, 4 * D)
        if Lk == a.L:
            qkv = torch.randn(1, a.L, 3 * D, device="cuda", generator=g).to(torch.bfloat16)
            q = k = v = qkv
            cols = (0, D, 2 * D)
        else:
            q = torch.randn(1, a.L, D, device="cuda", generator=g).to(torch.bfloat16)
            k = v = torch.randn(1, Lk, 2 * D, device="cuda", generator=g).to(torch.bfloat16)
            cols = (0, 0, D)
        o = torch.empty(1, a.L, D, dtype=torch.bfloat16, device="cuda")
        if a.fp8:
            # quantisation of q, k, v (five small kernels) included, as a caller sees it
            ws = torch.empty(wan.attention_fp8_workspace_bytes(cfg, 1, a.L, Lk), dtype=torch.uint8, device="cuda")
            ms = _time(lambda: wan.attention_fp8_fwd(cfg, q, k, v, o, a.heads, 128, *cols, 0, ws=ws), a.iters,
                       a.warmup)
        else:
            ws = None if a.no_split else torch.empty(max(16, wan.attention_workspace_bytes(cfg, 1, a.L)),
                                                     dtype=torch.uint8, device="cuda")
            ms = _time(lambda: wan.attention_fwd(cfg, q, k, v, o, a.heads, 128, *cols, 0, ws=ws), a.iters, a.warmup)
        flops = 4.0 * a.L * Lk * D
        out.update(L=a.L, Lk=Lk, heads=a.heads, split=not a.no_split, fp8=a.fp8, ms=ms, tflops=flops / ms / 1e9)
    elif a.kernel == "gemm":
        cfg = wan.make_config(128, 1, 128)
        A = torch.randn(a.M, a.K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(a.N, a.K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        bias = torch.zeros(a.N, dtype=torch.bfloat16, device="cuda")
        if a.epi in ("store", "gelu"):
            C = torch.empty(a.M, a.N, dtype=torch.bfloat16, device="cuda")
        else:
            C = torch.zeros(a.M, a.N, dtype=torch.float32, device="cuda")
        epi = {"store": wan.EPI_STORE, "gelu": wan.EPI_GELU, "residual": wan.EPI_RESIDUAL, "f32": wan.EPI_F32}[a.epi]
        if a.fp8:
            Aq = torch.empty(a.M, a.K, dtype=torch.uint8, device="cuda")
            As = torch.empty(a.M, dtype=torch.float32, device="cuda")
            Wq = torch.empty(a.N, a.K, dtype=torch.uint8, device="cuda")
            Ws = torch.empty(1, dtype=torch.float32, device="cuda")
            wan.fp8_quantize_rows(cfg, A, Aq, As)
            wan.fp8_quantize_tensor(cfg, W, Wq, Ws)
            del A, W
            ms = _time(lambda: wan.linear_fp8_fwd(cfg, Aq, As, Wq, Ws, bias, C, epi, rows_per_batch=a.M), a.iters,
                       a.warmup)
        else:
            ms = _time(lambda: wan.linear_fwd(cfg, A, W, bias, C, epi, rows_per_batch=a.M), a.iters, a.warmup)
        flops = 2.0 * a.M * a.N * a.K
        out.update(M=a.M, N=a.N, K=a.K, epi=a.epi, fp8=a.fp8, ms=ms, tflops=flops / ms / 1e9)
    elif a.kernel in ("patchify", "head"):
        out.update(_patch_or_head(a, g))
    elif a.kernel == "block":
        out.update(_block(a))
    elif a.kernel == "sample":
        out.update(_sample(a))
    else:
        cfg = wan.make_config(a.dim, a.dim // 64, a.dim)
        x = torch.randn(1, a.L, a.dim, device="cuda", generator=g)
        e = torch.randn(1, 6, a.dim, device="cuda", generator=g) * 0.1
        h = torch.empty(1, a.L, a.dim, dtype=torch.bfloat16, device="cuda")
        ms = _time(lambda: wan.adaln_modulate(cfg, x, e, None, 0, h), a.iters, a.warmup)
        byts = a.L * a.dim * 6.0
        out.update(L=a.L, dim=a.dim, ms=ms, gbs=byts / ms / 1e6)
    st = wan.device_status()
    out["status"] = wan.status_string(st)
    print(json.dumps(out), flush=True)
    return 0 if st == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
