"""Python binding of ``libwan_b200.so`` (the C ABI in ``include/wan.h``).

Argument marshalling only: every step of the Wan 2.1 DiT forward path runs in the
library's CUDA kernels. PyTorch supplies device memory and streams. Importing this
module is cheap; the first call loads the library and raises ImportError if it has not
been built (``python -m video_diffusion_transformer_wan_b200.build``). There is no
fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

__all__ = [
    "LIB_PATH", "lib", "WanError", "WAN_F32", "WAN_BF16", "EPI_STORE", "EPI_GELU", "EPI_RESIDUAL", "EPI_F32",
    "KIND_NORM", "KIND_GEMM", "KIND_ATTN", "KIND_SMALL", "Config", "BlockWeights", "TimeWeights", "ImageMlpWeights",
    "StackWeights", "DiffusionCache", "Fp8Scales", "make_config", "workspace_bytes", "device_status",
    "wait_timeout_check", "patchify", "patchify_noalloc", "time_mlp", "adaln_modulate", "self_attn_fwd",
    "cross_attn_fwd", "ffn_fwd", "dit_block_fwd", "dit_stack_fwd", "attention_fwd", "attention_workspace_bytes",
    "attention_fp8_fwd", "attention_fp8_quantize", "attention_fp8_workspace_bytes",
    "linear_fwd", "head_fwd", "i2v_input", "image_context_fwd", "flow_matching_input", "flow_matching_loss",
    "sample_workspace_bytes", "sample_euler_cfg", "sp_qkv_fwd", "sp_attn_fwd", "sp_out_fwd", "fp8_quantize_rows",
    "fp8_quantize_tensor", "linear_fp8_fwd", "fp8_workspace_bytes", "dit_block_fp8_fwd", "dit_stack_fp8_fwd",
    "launch_count", "trace_enable", "trace_reset", "trace_read", "trace_launches", "status_string",
]

LIB_PATH = os.environ.get("WAN_B200_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                            "libwan_b200.so")
WAN_F32, WAN_BF16 = 0, 1
EPI_STORE, EPI_GELU, EPI_RESIDUAL, EPI_F32 = 0, 1, 2, 3
KIND_NORM, KIND_GEMM, KIND_ATTN, KIND_SMALL = 0, 1, 2, 3

_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t


class Config(ctypes.Structure):
    _fields_ = [("dim", _i), ("heads", _i), ("head_dim", _i), ("ffn_dim", _i), ("in_ch", _i), ("out_ch", _i),
                ("freq_dim", _i), ("img_feat_dim", _i), ("eps", ctypes.c_float), ("dtype", _i)]


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ["mod_bias", "w_qkv", "b_qkv", "w_o", "b_o", "w_cq", "b_cq", "w_ckv", "b_ckv",
                                   "w_co", "b_co", "w_ckv_img", "b_ckv_img", "w_1", "b_1", "w_2", "b_2"]]


class TimeWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ["w_t1", "b_t1", "w_t2", "b_t2"]]


class ImageMlpWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ["w_1", "b_1", "w_2", "b_2", "w_3", "b_3"]]


class StackWeights(ctypes.Structure):
    _fields_ = [("w_p", _vp), ("b_p", _vp), ("time", TimeWeights), ("w_head", _vp), ("b_head", _vp)]


class DiffusionCache(ctypes.Structure):
    """Attention reuse and unconditional-pass skipping of the sampling loop (see
    ``wan_diffusion_cache`` in include/wan.h)."""
    _fields_ = [("attn_start", _i), ("attn_interval", _i), ("cfg_start", _i), ("cfg_interval", _i)]


class Fp8Scales(ctypes.Structure):
    """Device pointers of the per-tensor scales of a block's E4M3 weights; with
    attention_fp8 = 1 the block's self-attention also runs on E4M3 operands."""
    _fields_ = [(n, _vp) for n in ["qkv", "o", "cq", "ckv", "co", "ckv_img", "ffn1", "ffn2"]] + \
        [("attention_fp8", _i)]


class WanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m video_diffusion_transformer_wan_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    sig = {
        "wan_status_string": (ctypes.c_char_p, [_i]),
        "wan_workspace_bytes": (_sz, [P(Config), _i, _i, _i, _i]),
        "wan_device_status": (_i, [_vp]),
        "wan_wait_timeout_check": (_i, [_vp]),
        "wan_patchify": (_i, [P(Config), _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
        "wan_patchify_noalloc": (_i, [P(Config), _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
        "wan_time_mlp": (_i, [P(Config), _vp, _i, P(TimeWeights), _vp, _vp]),
        "wan_adaln_modulate": (_i, [P(Config), _vp, _i, _i, _vp, _vp, _i, _vp, _vp]),
        "wan_self_attn_fwd": (_i, [P(Config), _vp, P(BlockWeights), _vp, _vp, _i, _i, _vp, _sz, _vp]),
        "wan_cross_attn_fwd": (_i, [P(Config), _vp, _vp, _i, _vp, _i, P(BlockWeights), _vp, _i, _i, _vp, _sz, _vp]),
        "wan_ffn_fwd": (_i, [P(Config), _vp, P(BlockWeights), _vp, _vp, _i, _i, _vp, _sz, _vp]),
        "wan_dit_block_fwd": (_i, [P(Config), _vp, _vp, _vp, _i, _vp, _i, P(BlockWeights), _i, _i, _vp, _sz, _vp]),
        "wan_dit_stack_fwd": (_i, [P(Config), _i, _vp, _i, _i, _i, _i, _vp, P(StackWeights), P(BlockWeights), _vp,
                                   _i, _vp, _i, _vp, _vp, _sz, _vp]),
        "wan_head_fwd": (_i, [P(Config), _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
        "wan_i2v_input": (_i, [P(Config), _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
        "wan_image_context_fwd": (_i, [P(Config), _vp, _i, _i, P(ImageMlpWeights), _vp, _vp, _sz, _vp]),
        "wan_flow_matching_input": (_i, [P(Config), _vp, _vp, _vp, _i, _i64, _vp, _vp, _vp]),
        "wan_flow_matching_loss": (_i, [P(Config), _vp, _vp, _vp, _i, _i64, _vp, _vp]),
        "wan_attention_fwd": (_i, [P(Config), _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _i, _i,
                                   _i, _i, _i, _vp, _sz, _vp]),
        "wan_attention_workspace_bytes": (_sz, [P(Config), _i, _i]),
        "wan_attention_fp8_quantize": (_i, [P(Config), _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _i, _i, _i, _i,
                                            _i, _vp, _vp, _vp, _vp, _i64, _vp, _vp]),
        "wan_attention_fp8_fwd": (_i, [P(Config), _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _vp, _i64, _i, _i,
                                       _i, _i, _i, _i, _vp, _sz, _vp]),
        "wan_attention_fp8_workspace_bytes": (_sz, [P(Config), _i, _i, _i]),
        "wan_linear_fwd": (_i, [P(Config), _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _i64, _i, _vp]),
        "wan_sample_workspace_bytes": (_sz, [P(Config), _i, _i, _i, _i, _i, _i, _i, P(DiffusionCache), _i]),
        "wan_sample_euler_cfg": (_i, [P(Config), _i, _vp, _i, _i, _i, _i, _i, ctypes.c_float, P(StackWeights),
                                      P(BlockWeights), _vp, _vp, _i, _vp, _i, P(DiffusionCache), P(Fp8Scales), _vp,
                                      _vp, _sz, _vp]),
        "wan_dit_stack_fp8_fwd": (_i, [P(Config), _i, _vp, _i, _i, _i, _i, _vp, P(StackWeights), P(BlockWeights),
                                       P(Fp8Scales), _vp, _i, _vp, _i, _vp, _vp, _sz, _vp]),
        "wan_sp_qkv_fwd": (_i, [P(Config), _i, _i, _vp, _i, _i, P(BlockWeights), P(_vp), _vp]),
        "wan_sp_attn_fwd": (_i, [P(Config), _i, _i, _vp, _i, _i, P(_vp), _vp]),
        "wan_sp_out_fwd": (_i, [P(Config), _i, _vp, P(BlockWeights), _vp, _vp, _i, _i, _vp]),
        "wan_fp8_quantize_rows": (_i, [P(Config), _vp, _i, _i, _vp, _vp, _vp]),
        "wan_fp8_quantize_tensor": (_i, [P(Config), _vp, _i64, _vp, _vp, _vp]),
        "wan_linear_fp8_fwd": (_i, [P(Config), _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _i64, _i,
                                    _vp]),
        "wan_fp8_workspace_bytes": (_sz, [P(Config), _i, _i, _i, _i]),
        "wan_dit_block_fp8_fwd": (_i, [P(Config), _vp, _vp, _vp, _i, _vp, _i, P(BlockWeights), P(Fp8Scales), _i,
                                       _i, _vp, _sz, _vp]),
        "wan_launch_count": (_i64, []),
        "wan_trace_enable": (_i, [_i]),
        "wan_trace_reset": (_i, []),
        "wan_trace_read": (_i, [_i, P(ctypes.c_double), P(_i64)]),
        "wan_trace_launches": (_i, [_i, P(_i), P(ctypes.c_double), P(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


_LIB: Optional[ctypes.CDLL] = None


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return _lib()
    raise AttributeError(name)


def status_string(status: int) -> str:
    return _lib().wan_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise WanError(status, where)


def _p(t) -> Optional[int]:
    """Device pointer of a contiguous tensor (or None, or a raw address). The C calls take
    dense row-major arrays, so a strided view is refused here rather than misread."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got shape {tuple(t.shape)} strides {t.stride()}")
    return t.data_ptr()


def _p_strided(t) -> Optional[int]:
    """Device pointer of a tensor whose layout the call describes with explicit strides
    (the residual epilogue's gate rows)."""
    return None if t is None else (t if isinstance(t, int) else t.data_ptr())


def _stream(stream=None) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def make_config(dim: int, heads: int, ffn: int, in_ch: int = 16, out_ch: int = 16, freq_dim: int = 256,
                img_feat: int = 1280, eps: float = 1e-6, dtype: str = "bf16") -> Config:
    return Config(dim, heads, dim // heads, ffn, in_ch, out_ch, freq_dim, img_feat, eps,
                  WAN_BF16 if dtype == "bf16" else WAN_F32)


def block_weights(w: Dict[str, object]) -> BlockWeights:
    """Weight table from a dict of device tensors named as in ``BlockWeights``."""
    return BlockWeights(**{n: _p(w.get(n)) for n, _ in BlockWeights._fields_})


def workspace_bytes(cfg: Config, B: int, L: int, Lc: int, Li: int = 0) -> int:
    return int(_lib().wan_workspace_bytes(ctypes.byref(cfg), B, L, Lc, Li))


def device_status(stream=None) -> int:
    return int(_lib().wan_device_status(_stream(stream)))


def wait_timeout_check(stream=None) -> None:
    """Launch the one-thread kernel whose bounded wait runs out (about 1 s); the next
    device_status() returns WAN_ERR_TIMEOUT (-7)."""
    _check(_lib().wan_wait_timeout_check(_stream(stream)), "wan_wait_timeout_check")


def patchify(cfg, latent, w_p, b_p, x_out, ws, stream=None):
    B, C, F, H, W = latent.shape
    _check(_lib().wan_patchify(ctypes.byref(cfg), _p(latent), B, F, H, W, _p(w_p), _p(b_p), _p(x_out), _p(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "wan_patchify")


def patchify_noalloc(cfg, latent, w_p, b_p, x_out, stream=None):
    """wan_patchify without a workspace (fixed scratch inside the library)."""
    B, C, F, H, W = latent.shape
    _check(_lib().wan_patchify_noalloc(ctypes.byref(cfg), _p(latent), B, F, H, W, _p(w_p), _p(b_p), _p(x_out),
                                       _stream(stream)), "wan_patchify_noalloc")


def time_mlp(cfg, t, tw: TimeWeights, e_out, stream=None):
    _check(_lib().wan_time_mlp(ctypes.byref(cfg), _p(t), t.shape[0], ctypes.byref(tw), _p(e_out), _stream(stream)),
           "wan_time_mlp")


def adaln_modulate(cfg, x, e, mod_bias, chunk, h_out, stream=None):
    B, L, _ = x.shape
    _check(_lib().wan_adaln_modulate(ctypes.byref(cfg), _p(x), B, L, _p(e), _p(mod_bias), chunk, _p(h_out),
                                  _stream(stream)), "wan_adaln_modulate")


def _ws(ws):
    return (None, 0) if ws is None else (_p(ws), ws.numel() * ws.element_size())


def self_attn_fwd(cfg, h, bw: BlockWeights, e, x_inout, ws, stream=None):
    B, L, _ = x_inout.shape
    _check(_lib().wan_self_attn_fwd(ctypes.byref(cfg), _p(h), ctypes.byref(bw), _p(e), _p(x_inout), B, L, *_ws(ws),
                                 _stream(stream)), "wan_self_attn_fwd")


def cross_attn_fwd(cfg, h, ctx, img_ctx, bw: BlockWeights, x_inout, ws, stream=None):
    B, L, _ = x_inout.shape
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_cross_attn_fwd(ctypes.byref(cfg), _p(h), _p(ctx), ctx.shape[1], _p(img_ctx), Li,
                                  ctypes.byref(bw), _p(x_inout), B, L, *_ws(ws), _stream(stream)),
           "wan_cross_attn_fwd")


def ffn_fwd(cfg, h, bw: BlockWeights, e, x_inout, ws, stream=None):
    B, L, _ = x_inout.shape
    _check(_lib().wan_ffn_fwd(ctypes.byref(cfg), _p(h), ctypes.byref(bw), _p(e), _p(x_inout), B, L, *_ws(ws),
                           _stream(stream)), "wan_ffn_fwd")


def dit_block_fwd(cfg, x_inout, e, ctx, img_ctx, bw: BlockWeights, ws, stream=None):
    B, L, _ = x_inout.shape
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_dit_block_fwd(ctypes.byref(cfg), _p(x_inout), _p(e), _p(ctx), ctx.shape[1], _p(img_ctx), Li,
                                 ctypes.byref(bw), B, L, *_ws(ws), _stream(stream)), "wan_dit_block_fwd")


def dit_stack_fwd(cfg, latent, t, sw: StackWeights, blocks: Sequence[BlockWeights], ctx, img_ctx, v_out, ws,
                  stream=None):
    B, C, F, H, W = latent.shape
    arr = (BlockWeights * max(1, len(blocks)))(*blocks)
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_dit_stack_fwd(ctypes.byref(cfg), len(blocks), _p(latent), B, F, H, W, _p(t), ctypes.byref(sw),
                                 arr, _p(ctx), ctx.shape[1], _p(img_ctx), Li, _p(v_out), *_ws(ws), _stream(stream)),
           "wan_dit_stack_fwd")


def _cache_ref(cache: Optional[DiffusionCache]):
    return None if cache is None else ctypes.byref(cache)


def sample_workspace_bytes(cfg: Config, n_blocks: int, B: int, F: int, H: int, W: int, Lc: int, Li: int = 0,
                           cache: Optional[DiffusionCache] = None, fp8: bool = False) -> int:
    return int(_lib().wan_sample_workspace_bytes(ctypes.byref(cfg), n_blocks, B, F, H, W, Lc, Li, _cache_ref(cache),
                                                 1 if fp8 else 0))


def _scales_array(scales):
    return None if scales is None else (Fp8Scales * max(1, len(scales)))(*scales)


def sample_euler_cfg(cfg, inp, n_steps: int, guidance: float, sw: StackWeights, blocks: Sequence[BlockWeights],
                     ctx_cond, ctx_uncond, img_ctx, latent_out, ws, stream=None,
                     cache: Optional[DiffusionCache] = None, fp8_scales: Optional[Sequence[Fp8Scales]] = None):
    """inp [B, in_ch, F, H, W]: the noise in its first out_ch channels (and, for I2V, the
    fixed condition channels after them); latent_out [B, out_ch, F, H, W] fp32. With
    fp8_scales (one table per block) the blocks hold E4M3 codes."""
    B, C, F, H, W = inp.shape
    arr = (BlockWeights * max(1, len(blocks)))(*blocks)
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_sample_euler_cfg(ctypes.byref(cfg), len(blocks), _p(inp), B, F, H, W, n_steps, guidance,
                                    ctypes.byref(sw), arr, _p(ctx_cond), _p(ctx_uncond), ctx_cond.shape[1],
                                    _p(img_ctx), Li, _cache_ref(cache), _scales_array(fp8_scales),
                                    _p(latent_out), *_ws(ws), _stream(stream)),
           "wan_sample_euler_cfg")


def dit_stack_fp8_fwd(cfg, latent, t, sw: StackWeights, blocks: Sequence[BlockWeights],
                      scales: Sequence[Fp8Scales], ctx, img_ctx, v_out, ws, stream=None):
    """wan_dit_stack_fwd with E4M3 block weights (blocks: code tables, scales: one per block)."""
    B, C, F, H, W = latent.shape
    arr = (BlockWeights * max(1, len(blocks)))(*blocks)
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_dit_stack_fp8_fwd(ctypes.byref(cfg), len(blocks), _p(latent), B, F, H, W, _p(t),
                                     ctypes.byref(sw), arr, _scales_array(scales), _p(ctx), ctx.shape[1],
                                     _p(img_ctx), Li, _p(v_out), *_ws(ws), _stream(stream)),
           "wan_dit_stack_fp8_fwd")


def fp8_quantize_rows(cfg, x, q, scale, stream=None):
    """x [..., K] act -> q [..., K] uint8 (E4M3 codes), scale [rows] fp32."""
    K = x.shape[-1]
    _check(_lib().wan_fp8_quantize_rows(ctypes.byref(cfg), _p(x), x.numel() // K, K, _p(q), _p(scale),
                                     _stream(stream)), "wan_fp8_quantize_rows")


def fp8_quantize_tensor(cfg, x, q, scale, stream=None):
    """x act (any shape) -> q uint8 codes, scale [1] fp32 (one scale for the tensor)."""
    _check(_lib().wan_fp8_quantize_tensor(ctypes.byref(cfg), _p(x), x.numel(), _p(q), _p(scale),
                                       _stream(stream)), "wan_fp8_quantize_tensor")


def linear_fp8_fwd(cfg, A, a_scale, W, w_scale, bias, out, epilogue, gate=None, gate_bias=None,
                   gate_batch_stride=0, rows_per_batch=1, stream=None):
    K = A.shape[-1]
    M = A.numel() // K
    N = W.shape[0]
    _check(_lib().wan_linear_fp8_fwd(ctypes.byref(cfg), _p(A), _p(a_scale), _p(W), _p(w_scale), _p(bias), _p(out),
                                  M, N, K, epilogue, _p_strided(gate), _p(gate_bias), gate_batch_stride,
                                  rows_per_batch, _stream(stream)), "wan_linear_fp8_fwd")


def fp8_workspace_bytes(cfg: Config, B: int, L: int, Lc: int, Li: int = 0) -> int:
    return int(_lib().wan_fp8_workspace_bytes(ctypes.byref(cfg), B, L, Lc, Li))


def dit_block_fp8_fwd(cfg, x_inout, e, ctx, img_ctx, bw: BlockWeights, sc: Fp8Scales, ws, stream=None):
    B, L, _ = x_inout.shape
    Li = 0 if img_ctx is None else img_ctx.shape[1]
    _check(_lib().wan_dit_block_fp8_fwd(ctypes.byref(cfg), _p(x_inout), _p(e), _p(ctx), ctx.shape[1], _p(img_ctx),
                                     Li, ctypes.byref(bw), ctypes.byref(sc), B, L, *_ws(ws), _stream(stream)),
           "wan_dit_block_fp8_fwd")


def _ptr_table(bufs):
    return (_vp * len(bufs))(*[_p(b) for b in bufs])


def sp_qkv_fwd(cfg, sp_size: int, sp_rank: int, h, L: int, bw: BlockWeights, qkv_dst, stream=None):
    """h [B, L/P, D] (this rank's rows); qkv_dst: P buffers [B, L, 3D/P]."""
    _check(_lib().wan_sp_qkv_fwd(ctypes.byref(cfg), sp_size, sp_rank, _p(h), h.shape[0], L, ctypes.byref(bw),
                              _ptr_table(qkv_dst), _stream(stream)), "wan_sp_qkv_fwd")


def sp_attn_fwd(cfg, sp_size: int, sp_rank: int, qkv, L: int, o_dst, stream=None):
    """qkv [B, L, 3D/P] (this rank's heads); o_dst: P buffers [B, L/P, D]."""
    _check(_lib().wan_sp_attn_fwd(ctypes.byref(cfg), sp_size, sp_rank, _p(qkv), qkv.shape[0], L,
                               _ptr_table(o_dst), _stream(stream)), "wan_sp_attn_fwd")


def sp_out_fwd(cfg, sp_size: int, o, bw: BlockWeights, e, x_inout, L: int, stream=None):
    """o [B, L/P, D] act, x_inout [B, L/P, D] fp32, e [B, 6, D] fp32."""
    _check(_lib().wan_sp_out_fwd(ctypes.byref(cfg), sp_size, _p(o), ctypes.byref(bw), _p(e), _p(x_inout),
                              o.shape[0], L, _stream(stream)), "wan_sp_out_fwd")


def attention_workspace_bytes(cfg: Config, B: int, Lq: int) -> int:
    return int(_lib().wan_attention_workspace_bytes(ctypes.byref(cfg), B, Lq))


def attention_fwd(cfg, q, k, v, o, heads, head_dim, q_col0=0, k_col0=0, v_col0=0, o_col0=0, stream=None, ws=None):
    """q [B, Lq, *], k/v [B, Lk, *], o [B, Lq, *] (contiguous rows); ws: optional scratch
    of attention_workspace_bytes (lets a last partial wave split over the keys)."""
    B, Lq, qs = q.shape
    Lk, ks = k.shape[1], k.shape[2]
    _check(_lib().wan_attention_fwd(ctypes.byref(cfg), _p(q), qs, q_col0, _p(k), ks, k_col0, _p(v), v.shape[2], v_col0,
                                 _p(o), o.shape[2], o_col0, B, heads, Lq, Lk, head_dim, *_ws(ws), _stream(stream)),
           "wan_attention_fwd")


def attention_fp8_workspace_bytes(cfg: Config, B: int, Lq: int, Lk: int) -> int:
    return int(_lib().wan_attention_fp8_workspace_bytes(ctypes.byref(cfg), B, Lq, Lk))


def attention_fp8_fwd(cfg, q, k, v, o, heads, head_dim, q_col0=0, k_col0=0, v_col0=0, o_col0=0, ws=None,
                      stream=None):
    """8-bit attention: the operands of attention_fwd; ws (required) of
    attention_fp8_workspace_bytes holds the E4M3 codes and scales."""
    B, Lq, qs = q.shape
    Lk, ks = k.shape[1], k.shape[2]
    _check(_lib().wan_attention_fp8_fwd(ctypes.byref(cfg), _p(q), qs, q_col0, _p(k), ks, k_col0, _p(v), v.shape[2],
                                     v_col0, _p(o), o.shape[2], o_col0, B, heads, Lq, Lk, head_dim, *_ws(ws),
                                     _stream(stream)), "wan_attention_fp8_fwd")


def attention_fp8_quantize(cfg, q, k, v, heads, head_dim, q_codes, q_scale, k_codes, vt_codes, kv_scale, q_col0=0,
                           k_col0=0, v_col0=0, stream=None):
    """E4M3 operands of attention_fp8_fwd into caller tensors: q_codes [B, Lq, H*d] and
    k_codes [B, Lk, H*d] uint8, vt_codes [B, H*d, S] uint8 (S % 64 == 0, S >= Lk),
    q_scale [B, Lq, H] and kv_scale [B, H, 2] float32."""
    B, Lq, qs = q.shape
    Lk, ks = k.shape[1], k.shape[2]
    _check(_lib().wan_attention_fp8_quantize(ctypes.byref(cfg), _p(q), qs, q_col0, _p(k), ks, k_col0, _p(v),
                                          v.shape[2], v_col0, B, heads, Lq, Lk, head_dim, _p(q_codes), _p(q_scale),
                                          _p(k_codes), _p(vt_codes), vt_codes.shape[2], _p(kv_scale),
                                          _stream(stream)), "wan_attention_fp8_quantize")


def linear_fwd(cfg, A, W, bias, out, epilogue, gate=None, gate_bias=None, gate_batch_stride=0, rows_per_batch=1,
               stream=None):
    K = A.shape[-1]
    M = A.numel() // K
    N = W.shape[0]
    _check(_lib().wan_linear_fwd(ctypes.byref(cfg), _p(A), _p(W), _p(bias), _p(out), M, N, K, epilogue,
                              _p_strided(gate), _p(gate_bias), gate_batch_stride, rows_per_batch, _stream(stream)),
           "wan_linear_fwd")


def head_fwd(cfg, x, F, H, W, w_head, b_head, v_out, ws, stream=None):
    B = x.shape[0]
    _check(_lib().wan_head_fwd(ctypes.byref(cfg), _p(x), B, F, H, W, _p(w_head), _p(b_head), _p(v_out), *_ws(ws),
                            _stream(stream)), "wan_head_fwd")


def i2v_input(cfg, noise, cond, frame_keep, out, stream=None):
    B, C, F, H, W = noise.shape
    _check(_lib().wan_i2v_input(ctypes.byref(cfg), _p(noise), _p(cond), _p(frame_keep), B, F, H, W, _p(out),
                             _stream(stream)), "wan_i2v_input")


def image_context_fwd(cfg, feat, iw: ImageMlpWeights, out, ws, stream=None):
    B, Li, _ = feat.shape
    _check(_lib().wan_image_context_fwd(ctypes.byref(cfg), _p(feat), B, Li, ctypes.byref(iw), _p(out), *_ws(ws),
                                     _stream(stream)), "wan_image_context_fwd")


def flow_matching_input(cfg, x1, x0, u, xt_out, t_out, stream=None):
    B = x1.shape[0]
    _check(_lib().wan_flow_matching_input(ctypes.byref(cfg), _p(x1), _p(x0), _p(u), B, x1.numel() // B, _p(xt_out),
                                       _p(t_out), _stream(stream)), "wan_flow_matching_input")


def flow_matching_loss(cfg, v, x1, x0, loss_out, stream=None):
    B = x1.shape[0]
    _check(_lib().wan_flow_matching_loss(ctypes.byref(cfg), _p(v), _p(x1), _p(x0), B, x1.numel() // B, _p(loss_out),
                                      _stream(stream)), "wan_flow_matching_loss")


def launch_count() -> int:
    return int(_lib().wan_launch_count())


def trace_enable(on: bool = True) -> None:
    _check(_lib().wan_trace_enable(1 if on else 0), "wan_trace_enable")


def trace_reset() -> None:
    _check(_lib().wan_trace_reset(), "wan_trace_reset")


def trace_launches(cap: int = 16384):
    """Per-launch (kind, ms, work) records since the last reset."""
    kinds = (_i * cap)()
    ms = (ctypes.c_double * cap)()
    work = (ctypes.c_double * cap)()
    n = _lib().wan_trace_launches(cap, kinds, ms, work)
    if n < 0:
        raise WanError(n, "wan_trace_launches")
    return [(kinds[i], ms[i], work[i]) for i in range(n)]


def trace_read(kind: int):
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    _check(_lib().wan_trace_read(kind, ctypes.byref(ms), ctypes.byref(n)), "wan_trace_read")
    return ms.value, n.value
