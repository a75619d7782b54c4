"""Single-kernel micro-benchmark through the C ABI (CUDA-event timing), also the
command the committed ncu summaries were captured with.

  python -m video_diffusion_transformer_wan_b200.kernel_bench attention --L 32760 --heads 12
  python -m video_diffusion_transformer_wan_b200.kernel_bench gemm --M 32760 --N 4608 --K 1536 --epi store
  python -m video_diffusion_transformer_wan_b200.kernel_bench layernorm --L 32760 --dim 1536

Inputs are random device tensors (the kernels' timing does not depend on values).
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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["attention", "gemm", "layernorm"])
    ap.add_argument("--L", type=int, default=32760)
    ap.add_argument("--Lk", type=int, default=0, help="key length (default: L, self-attention)")
    ap.add_argument("--heads", type=int, default=12)
    ap.add_argument("--dim", type=int, default=1536)
    ap.add_argument("--M", type=int, default=32760)
    ap.add_argument("--N", type=int, default=4608)
    ap.add_argument("--K", type=int, default=1536)
    ap.add_argument("--epi", choices=["store", "gelu", "residual", "f32"], default="store")
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
        ms = _time(lambda: wan.attention_fwd(cfg, q, k, v, o, a.heads, 128, *cols, 0), a.iters, a.warmup)
        flops = 4.0 * a.L * Lk * D
        out.update(L=a.L, Lk=Lk, heads=a.heads, ms=ms, tflops=flops / ms / 1e9)
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
        ms = _time(lambda: wan.linear_fwd(cfg, A, W, bias, C, epi, rows_per_batch=a.M), a.iters, a.warmup)
        flops = 2.0 * a.M * a.N * a.K
        out.update(M=a.M, N=a.N, K=a.K, epi=a.epi, ms=ms, tflops=flops / ms / 1e9)
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
