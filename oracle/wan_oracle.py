"""CPU oracle for the Wan 2.1 DiT forward hot path.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
definition the CUDA library is checked against. Only the tests, the smoke check
and the benchmark's CPU-baseline leg may import it; the library never calls it
and shares no code with it.

Every function works in float64 on one sample (no batch axis) and writes the
definition out directly, with numpy matmul as the only library step. Sources are
the pages on Wan 2.1:

* [Wan-P2] "Wan: Open and Advanced Large-Scale Video Generative Models (Wan 2.1)",
  zhao9797.github.io, sections "Diffusion Transformer", "I2V 架构扩展" (I2V
  extension), "训练方法" (training method) and the config table.
* [Wan-P1] "超越Sora！阿里正式完全开源 ... Wan2.1", 163.com, sections
  "核心创新二" (DiT) and "核心创新四" (I2V).

Where the pages are silent the plainest reading is taken; each such reading is
named in the docstring ("reading: ...").

Parity-pin status: every function here is pinned by a ``-m "not gpu"`` test
against something other than itself (a library routine, a closed form, an
invariant, or brute force). None is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

F64 = np.float64


def _f(a) -> np.ndarray:
    return np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------------------
# Shapes
# --------------------------------------------------------------------------------------

def token_count(latent_frames: int, latent_h: int, latent_w: int) -> int:
    """Sequence length after the (1,2,2) patchify [Wan-P2, "Diffusion Transformer"]:
    L = (1+T/4) * H/16 * W/16 in pixel units; the latent grid is already H/8 x W/8
    (Wan-VAE 4x8x8 compression, [Wan-P2, "Wan-VAE"]), so L = F * (h/2) * (w/2)."""
    if latent_h % 2 or latent_w % 2:
        raise ValueError("latent height and width must be even for (1,2,2) patches")
    return latent_frames * (latent_h // 2) * (latent_w // 2)


# --------------------------------------------------------------------------------------
# Patchify / unpatchify  [Wan-P2, "Diffusion Transformer": patchify is a 3D convolution
# with kernel (1,2,2); the sequence is unpatchified at the end]
# --------------------------------------------------------------------------------------

def patchify(latent, weight, bias) -> np.ndarray:
    """3D convolution with kernel = stride = (1,2,2) over ``latent [C,F,H,W]`` with
    ``weight [D,C,1,2,2]`` and ``bias [D]``, returning tokens ``[L,D]``.

    Because the kernel equals the stride the patches do not overlap, so the
    convolution is exactly: for every output position (f,i,j),
    ``x[(f,i,j), d] = bias[d] + sum_{c,ph,pw} weight[d,c,0,ph,pw] * latent[c,f,2i+ph,2j+pw]``.
    reading: tokens are ordered (f, i, j) row-major; the weight is flattened in
    (c, ph, pw) order with pw fastest (the natural layout of the conv weight)."""
    lat = _f(latent)
    w = _f(weight)
    C, F, H, W = lat.shape
    D = w.shape[0]
    assert w.shape == (D, C, 1, 2, 2)
    patches = lat.reshape(C, F, H // 2, 2, W // 2, 2)          # c, f, i, ph, j, pw
    patches = patches.transpose(1, 2, 4, 0, 3, 5)               # f, i, j, c, ph, pw
    patches = patches.reshape(F * (H // 2) * (W // 2), C * 4)
    return patches @ w.reshape(D, C * 4).T + _f(bias)[None, :]


def unpatchify(tokens, out_ch: int, frames: int, height: int, width: int) -> np.ndarray:
    """Inverse of the patch gather: ``tokens [L, out_ch*4]`` laid out (c, ph, pw) per
    token, tokens ordered (f, i, j), back to ``[out_ch, F, H, W]``
    [Wan-P2, "Diffusion Transformer": patchify -> blocks -> unpatchify]."""
    y = _f(tokens)
    hi, wi = height // 2, width // 2
    y = y.reshape(frames, hi, wi, out_ch, 2, 2)                  # f, i, j, c, ph, pw
    y = y.transpose(3, 0, 1, 4, 2, 5)                            # c, f, i, ph, j, pw
    return y.reshape(out_ch, frames, height, width)


# --------------------------------------------------------------------------------------
# Timestep embedding and the shared AdaLN MLP
# --------------------------------------------------------------------------------------

def sinusoidal_embedding(t: float, dim: int = 256) -> np.ndarray:
    """Sinusoidal timestep embedding; the frequency dimension is 256 [Wan-P2, note under
    the config table]. reading: frequencies 10000^(-i/(dim/2)) for i < dim/2, cosines
    first, then sines (the DiT lineage the page cites)."""
    half = dim // 2
    freqs = np.power(F64(10000.0), -np.arange(half, dtype=F64) / half)
    args = F64(t) * freqs
    return np.concatenate([np.cos(args), np.sin(args)])


def silu(x) -> np.ndarray:
    x = _f(x)
    return x / (1.0 + np.exp(-x))


def linear(x, weight, bias=None) -> np.ndarray:
    """y = x W^T + b with ``weight [out, in]``."""
    y = _f(x) @ _f(weight).T
    if bias is not None:
        y = y + _f(bias)
    return y


def time_mlp(t: float, w1, b1, w2, b2, freq_dim: int = 256) -> np.ndarray:
    """Shared timestep MLP: one MLP of Linear + SiLU layers predicts the six
    modulation vectors and is shared by all blocks [Wan-P2, "Diffusion Transformer";
    Wan-P1, "核心创新二"]. reading: sinusoid(256) -> Linear(256,D) -> SiLU ->
    Linear(D,6D), reshaped to ``[6, D]``."""
    e = sinusoidal_embedding(t, freq_dim)
    hdn = silu(linear(e, w1, b1))
    out = linear(hdn, w2, b2)
    return out.reshape(6, -1)


def block_modulation(e, mod_bias) -> np.ndarray:
    """Each block learns its own bias on top of the shared MLP output
    [Wan-P2, "Diffusion Transformer"; Wan-P1, "核心创新二"]: ``mod = e + bias_b``.
    reading: rows are (shift_msa, scale_msa, gate_msa, shift_ffn, scale_ffn, gate_ffn)."""
    return _f(e) + _f(mod_bias)


# --------------------------------------------------------------------------------------
# Normalisation, activation, attention
# --------------------------------------------------------------------------------------

def layer_norm(x, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm over the last axis without affine parameters, biased variance
    (divide by D), eps = 1e-6."""
    x = _f(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(h, shift, scale) -> np.ndarray:
    """AdaLN modulation. reading: ``h * (1 + scale) + shift`` (DiT convention)."""
    return _f(h) * (1.0 + _f(scale)) + _f(shift)


def gelu_tanh(x) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = _f(x)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def softmax(s, axis: int = -1) -> np.ndarray:
    s = _f(s)
    z = np.exp(s - s.max(axis=axis, keepdims=True))
    return z / z.sum(axis=axis, keepdims=True)


def attention(q, k, v, heads: int) -> np.ndarray:
    """Multi-head scaled dot-product attention, non-causal, no dropout: per head,
    ``softmax(q k^T / sqrt(d)) v`` with heads as contiguous d-wide slices of the model
    width. Used for the full spatio-temporal self-attention [Wan-P2, "Diffusion
    Transformer": full spatio-temporal attention] and the text cross-attention
    [Wan-P1, "核心创新二": cross-attention in every block]. reading: no positional
    encoding and no q/k normalisation (the pages mention neither)."""
    q, k, v = _f(q), _f(k), _f(v)
    Lq, D = q.shape
    d = D // heads
    out = np.empty((Lq, D), dtype=F64)
    step = 512  # query rows are independent; this bound only limits memory
    for hh in range(heads):
        sl = slice(hh * d, (hh + 1) * d)
        for r0 in range(0, Lq, step):
            p = softmax(q[r0:r0 + step, sl] @ k[:, sl].T / math.sqrt(d), axis=-1)
            out[r0:r0 + step, sl] = p @ v[:, sl]
    return out


# --------------------------------------------------------------------------------------
# Block branches
# --------------------------------------------------------------------------------------

def self_attention_core(h, w: Dict[str, np.ndarray], heads: int, kv_source=None, fp8: bool = False,
                        fp8_attention: bool = False) -> np.ndarray:
    """The attention output ``attn(h Wq, h Wk, h Wv)`` before the output projection.
    The fused QKV weight ``w_qkv [3D, D]`` is stacked (q, k, v). ``kv_source`` (all rows
    of h) lets the caller evaluate only some query rows; by default it is ``h``. With
    ``fp8`` the projection is ``linear_fp8`` of the fused weight (one weight scale); with
    ``fp8_attention`` the attention is ``attention_fp8`` (its q scales are per row, its
    k and v scales over all key rows, so a subset of query rows stays exact)."""
    attn = attention_fp8 if fp8_attention else attention
    h = _f(h)
    D = h.shape[-1]
    src = h if kv_source is None else _f(kv_source)
    wqkv, bqkv = _f(w["w_qkv"]), _f(w["b_qkv"])
    if fp8:
        q = linear_fp8(h, wqkv, bqkv)[:, :D]
        kv = linear_fp8(src, wqkv, bqkv)
        return attn(q, kv[:, D:2 * D], kv[:, 2 * D:], heads)
    q = linear(h, wqkv[:D], bqkv[:D])
    k = linear(src, wqkv[D:2 * D], bqkv[D:2 * D])
    v = linear(src, wqkv[2 * D:], bqkv[2 * D:])
    return attn(q, k, v, heads)


def self_attention_branch(h, w: Dict[str, np.ndarray], heads: int,
                          kv_source=None, o=None, fp8: bool = False) -> np.ndarray:
    """Self-attention sub-layer output before the gate: ``attn(h Wq, h Wk, h Wv) Wo^T + bo``.
    ``o`` replaces the attention output when given (an output kept from an earlier
    sampling step, see ``dit_block``'s ``attn_cache``)."""
    if o is None:
        o = self_attention_core(h, w, heads, kv_source, fp8)
    return (linear_fp8 if fp8 else linear)(o, w["w_o"], w["b_o"])


def cross_attention_branch(h, ctx, w: Dict[str, np.ndarray], heads: int,
                           img_ctx=None, fp8: bool = False) -> np.ndarray:
    """Cross-attention sub-layer: queries from the video tokens, keys and values from
    the 512 umT5 text tokens [Wan-P2, "Diffusion Transformer" and "umT5"]. For I2V, a
    decoupled second attention over image-context tokens with its own K/V projection
    is added before the shared output projection [Wan-P2, "I2V 架构扩展"; Wan-P1,
    "核心创新四"]. reading: ``o = attn(q,Kt,Vt) + attn(q,Ki,Vi)``, weight 1."""
    lin = linear_fp8 if fp8 else linear
    D = _f(h).shape[-1]
    q = lin(h, w["w_cq"], w["b_cq"])
    kv = lin(ctx, w["w_ckv"], w["b_ckv"])
    o = attention(q, kv[:, :D], kv[:, D:], heads)
    if img_ctx is not None:
        kvi = lin(img_ctx, w["w_ckv_img"], w["b_ckv_img"])
        o = o + attention(q, kvi[:, :D], kvi[:, D:], heads)
    return lin(o, w["w_co"], w["b_co"])


def ffn_branch(h, w: Dict[str, np.ndarray], fp8: bool = False) -> np.ndarray:
    """Feed-forward sub-layer: Linear(D,F) -> GELU-tanh -> Linear(F,D)
    [Wan-P2 config table: FFN dimension 8960 / 13824]. reading: a plain two-matrix
    FFN (a gated GLU would not match the 1.3B/14B parameter counts)."""
    lin = linear_fp8 if fp8 else linear
    return lin(gelu_tanh(lin(h, w["w_1"], w["b_1"])), w["w_2"], w["b_2"])


def dit_block(x, e, w: Dict[str, np.ndarray], ctx, heads: int, eps: float = 1e-6,
              img_ctx=None, rows: Optional[Sequence[int]] = None,
              return_parts: bool = False, attn_cache: Optional[Dict] = None, fp8: bool = False,
              fp8_attention: bool = False):
    """One DiT block [Wan-P2, "Diffusion Transformer"]:

    1. ``x += gate_msa * SelfAttn(LN(x) (1 + scale_msa) + shift_msa)``
    2. ``x += CrossAttn(LN(x), ctx[, img_ctx])``
    3. ``x += gate_ffn * FFN(LN(x) (1 + scale_ffn) + shift_ffn)``

    with ``mod = e + mod_bias`` (six vectors, see ``block_modulation``).
    reading: self-attention, then cross-attention, then FFN; the cross-attention
    input gets a plain LayerNorm and its residual has no gate (the pages give six
    modulation vectors, i.e. two gated branches).

    ``rows`` evaluates only those query rows; it is exact because every step but
    self-attention is row-local, and self-attention still takes keys and values from
    all rows. Returns ``x_out`` (of the selected rows), and with ``return_parts``
    also a dict of intermediates for those rows.

    ``attn_cache`` (the attention cache of a sampling loop, see
    ``sample_euler_cfg_cached``): a dict whose ``"o"`` holds this block's last computed
    attention output. With ``attn_cache["reuse"]`` true that output replaces the
    attention (q, k and v are not formed); otherwise the attention is computed and
    stored in ``attn_cache["o"]``.

    ``fp8`` runs every linear layer of the block as ``linear_fp8`` (per-token input
    codes, per-tensor weight codes; the sum of the text and image attention outputs is
    quantised as one input); ``fp8_attention`` also runs the self-attention as
    ``attention_fp8`` (the cross-attention keeps exact attention).
    """
    x = _f(x)
    mod = block_modulation(e, w["mod_bias"])
    shift_msa, scale_msa, gate_msa, shift_ffn, scale_ffn, gate_ffn = mod
    h_all = modulate(layer_norm(x, eps), shift_msa, scale_msa)
    if rows is None:
        xr, hr = x, h_all
    else:
        rows = np.asarray(rows)
        xr, hr = x[rows], h_all[rows]
    parts = {"h_msa": hr}
    if attn_cache is not None and attn_cache.get("reuse"):
        sa = self_attention_branch(hr, w, heads, o=attn_cache["o"], fp8=fp8)
    else:
        o = self_attention_core(hr, w, heads, kv_source=h_all, fp8=fp8, fp8_attention=fp8_attention)
        if attn_cache is not None:
            attn_cache["o"] = o
        sa = self_attention_branch(hr, w, heads, o=o, fp8=fp8)
    parts["sa"] = sa
    x1 = xr + gate_msa * sa
    hc = layer_norm(x1, eps)
    parts["h_cross"] = hc
    ca = cross_attention_branch(hc, ctx, w, heads, img_ctx=img_ctx, fp8=fp8)
    parts["ca"] = ca
    x2 = x1 + ca
    hf = modulate(layer_norm(x2, eps), shift_ffn, scale_ffn)
    parts["h_ffn"] = hf
    ff = ffn_branch(hf, w, fp8=fp8)
    parts["ffn"] = ff
    x3 = x2 + gate_ffn * ff
    parts["x_after_sa"], parts["x_after_ca"] = x1, x2
    return (x3, parts) if return_parts else x3


# --------------------------------------------------------------------------------------
# I2V input fusion and image context  [Wan-P2, "I2V 架构扩展"; Wan-P1, "核心创新四"]
# --------------------------------------------------------------------------------------

def i2v_mask(frame_keep, latent_frames: int, height: int, width: int,
             temporal_stride: int = 4) -> np.ndarray:
    """Binary mask (1 = keep, 0 = generate) over the pixel frames, reshaped to the VAE
    temporal stride. reading: the first pixel frame's value is repeated ``stride``
    times so the 1+T frames become ``latent_frames * stride`` values, which are
    grouped as ``[latent_frames, stride]`` and put on the channel axis, giving
    ``[stride, F, H, W]`` broadcast over the latent grid."""
    m = np.asarray(frame_keep, dtype=F64).reshape(-1)
    assert m.shape[0] == 1 + temporal_stride * (latent_frames - 1)
    m = np.concatenate([np.repeat(m[:1], temporal_stride), m[1:]])
    m = m.reshape(latent_frames, temporal_stride).T                  # [stride, F]
    return np.broadcast_to(m[:, :, None, None], (temporal_stride, latent_frames, height, width)).copy()


def i2v_input(noise, cond, mask) -> np.ndarray:
    """Noise latent, condition latent and reshaped mask concatenated on channels."""
    return np.concatenate([_f(noise), _f(cond), _f(mask)], axis=0)


def image_context_mlp(feat, w1, b1, w2, b2, w3, b3) -> np.ndarray:
    """Three-layer MLP projecting image-encoder features to the global image context.
    reading: Linear(1280,D) -> GELU-tanh -> Linear(D,D) -> GELU-tanh -> Linear(D,D)."""
    hdn = gelu_tanh(linear(feat, w1, b1))
    hdn = gelu_tanh(linear(hdn, w2, b2))
    return linear(hdn, w3, b3)


# --------------------------------------------------------------------------------------
# Head, stack and flow matching
# --------------------------------------------------------------------------------------

def head(x, w_head, b_head, eps: float = 1e-6) -> np.ndarray:
    """Output head. reading: plain LayerNorm, then Linear(D, out_ch*4)."""
    return linear(layer_norm(x, eps), w_head, b_head)


def flow_matching_input(x1, x0, u: float) -> np.ndarray:
    """Intermediate latent of rectified flow [Wan-P2, "训练方法"]: x_t = t x1 + (1-t) x0."""
    return F64(u) * _f(x1) + (1.0 - F64(u)) * _f(x0)


def flow_matching_target(x1, x0) -> np.ndarray:
    """Ground-truth velocity v_t = x1 - x0 [Wan-P2, "训练方法"]."""
    return _f(x1) - _f(x0)


def dit_stack(latent, t: float, weights: Dict, blocks: Sequence[Dict], ctx, heads: int,
              eps: float = 1e-6, img_ctx=None, freq_dim: int = 256,
              attn_caches: Optional[Sequence[Dict]] = None, fp8: bool = False,
              fp8_attention: bool = False) -> np.ndarray:
    """Whole DiT on one sample [Wan-P2, "Diffusion Transformer"]: patchify -> the time
    MLP shared by all blocks -> N blocks (each with its own modulation bias) -> head ->
    unpatchify. ``weights`` holds ``w_p, b_p, w_t1, b_t1, w_t2, b_t2, w_head, b_head``.
    ``attn_caches`` gives each block its attention cache (see ``dit_block``); ``fp8``
    runs the blocks' linear layers in FP8 and ``fp8_attention`` their self-attention
    (``dit_block``; patchify, the time MLP and the head stay as they are). Returns the
    predicted velocity ``[out_ch, F, H, W]``."""
    lat = _f(latent)
    C, F, H, W = lat.shape
    x = patchify(lat, weights["w_p"], weights["b_p"])
    e = time_mlp(t, weights["w_t1"], weights["b_t1"], weights["w_t2"], weights["b_t2"], freq_dim)
    for i, blk in enumerate(blocks):
        x = dit_block(x, e, blk, ctx, heads, eps, img_ctx=img_ctx,
                      attn_cache=None if attn_caches is None else attn_caches[i], fp8=fp8,
                      fp8_attention=fp8_attention)
    y = head(x, weights["w_head"], weights["b_head"], eps)
    return unpatchify(y, _f(weights["w_head"]).shape[0] // 4, F, H, W)


# --------------------------------------------------------------------------------------
# Sampling: rectified-flow Euler integration with classifier-free guidance
# [Wan-P2, "Infra": about 50 sampling steps; "训练方法": the model predicts the velocity
# x1 - x0 along x_t = t x1 + (1 - t) x0, noise at t = 0]
# --------------------------------------------------------------------------------------

def euler_cfg(x0, n_steps: int, guidance: float, velocity_cond, velocity_uncond) -> np.ndarray:
    """Integrate dx/dt = v(x, t) from t = 0 (noise) to t = 1 with ``n_steps`` Euler
    steps on the uniform grid t_k = k / n_steps, where the velocity is the guided
    combination ``v_u + guidance * (v_c - v_u)`` of the conditional and unconditional
    predictions ``velocity_*(x, t_k)``. reading: uniform grid in t, explicit Euler,
    guidance applied to the velocity (the pages give only the step count and a
    guidance scale)."""
    x = _f(x0).copy()
    dt = 1.0 / n_steps
    for k in range(n_steps):
        t = k * dt
        vc = _f(velocity_cond(x, t))
        vu = _f(velocity_uncond(x, t))
        x = x + dt * (vu + guidance * (vc - vu))
    return x


def sample_euler_cfg(noise, n_steps: int, guidance: float, weights: Dict, blocks: Sequence[Dict], ctx_cond,
                     ctx_uncond, heads: int, eps: float = 1e-6, img_ctx=None, cond_channels=None,
                     freq_dim: int = 256, fp8: bool = False, fp8_attention: bool = False) -> np.ndarray:
    """Generate a latent with the DiT as the velocity model: ``euler_cfg`` with
    ``v(x, t) = dit_stack(input(x), 1000 t, ...)`` under the text context (conditional)
    and the unconditional context. ``noise [16, F, H, W]`` is x at t = 0. For I2V,
    ``cond_channels [20, F, H, W]`` (condition latent and mask) are appended to x on the
    channel axis at every step and stay fixed. reading: the image context is used by
    both branches; only the text context differs."""
    def make_input(x):
        return x if cond_channels is None else np.concatenate([x, _f(cond_channels)], axis=0)

    def vel(ctx):
        return lambda x, t: dit_stack(make_input(x), 1000.0 * t, weights, blocks, ctx, heads, eps,
                                      img_ctx=img_ctx, freq_dim=freq_dim, fp8=fp8, fp8_attention=fp8_attention)
    return euler_cfg(noise, n_steps, guidance, vel(ctx_cond), vel(ctx_uncond))


# --------------------------------------------------------------------------------------
# Diffusion cache  [Wan-P2, "Infra", inference optimisation: (1) a block's attention
# output changes little from one sampling step to the next, so it is computed every few
# steps and reused in between; (2) late in sampling the conditional and unconditional
# predictions are close, so the unconditional pass is skipped and replaced by the
# conditional one corrected by a kept residual]
# --------------------------------------------------------------------------------------

def diffusion_cache_schedule(n_steps: int, attn_start: int, attn_interval: int, cfg_start: int,
                             cfg_interval: int):
    """Per sampling step k, ``(reuse_attention, skip_unconditional)``. reading: before
    ``attn_start`` every step computes attention; from it on, steps
    ``attn_start + m * attn_interval`` compute it and the others reuse each block's
    last output (``attn_interval = 1``: never reuse). The unconditional pass follows
    the same rule with ``cfg_start`` and ``cfg_interval``. Step 0 always computes
    both (``*_start >= 1`` or a computing step at 0)."""
    out = []
    for k in range(n_steps):
        ra = k >= attn_start and (k - attn_start) % attn_interval != 0
        su = k >= cfg_start and (k - cfg_start) % cfg_interval != 0
        out.append((ra, su))
    return out


def euler_cfg_cached(x0, n_steps: int, guidance: float, velocity_cond, velocity_uncond, schedule) -> np.ndarray:
    """``euler_cfg`` with the diffusion cache. ``velocity_*(x, t, reuse_attention)``.
    On a step that skips the unconditional pass, the guided velocity is
    ``v_c + (guidance - 1) * delta`` with ``delta = v_c - v_u`` kept from the last step
    that ran both passes. reading: the residual compensation is that kept difference
    (the unconditional prediction is taken as ``v_c - delta``)."""
    x = _f(x0).copy()
    dt = 1.0 / n_steps
    delta = None
    for k in range(n_steps):
        t = k * dt
        reuse, skip = schedule[k]
        vc = _f(velocity_cond(x, t, reuse))
        if skip:
            v = vc + (guidance - 1.0) * delta
        else:
            vu = _f(velocity_uncond(x, t, reuse))
            delta = vc - vu
            v = vu + guidance * delta
        x = x + dt * v
    return x


def sample_euler_cfg_cached(noise, n_steps: int, guidance: float, weights: Dict, blocks: Sequence[Dict], ctx_cond,
                            ctx_uncond, heads: int, schedule, eps: float = 1e-6, img_ctx=None, cond_channels=None,
                            freq_dim: int = 256, fp8: bool = False, fp8_attention: bool = False) -> np.ndarray:
    """``sample_euler_cfg`` with the diffusion cache of ``schedule``
    (``diffusion_cache_schedule``). Each branch keeps its own per-block attention
    outputs: a branch that reuses attention takes the outputs of the last step on which
    that branch computed it. ``fp8`` / ``fp8_attention`` as in ``dit_stack``."""
    caches = {"c": [{} for _ in blocks], "u": [{} for _ in blocks]}

    def make_input(x):
        return x if cond_channels is None else np.concatenate([x, _f(cond_channels)], axis=0)

    def vel(ctx, key):
        def f(x, t, reuse):
            for c in caches[key]:
                c["reuse"] = reuse
            return dit_stack(make_input(x), 1000.0 * t, weights, blocks, ctx, heads, eps, img_ctx=img_ctx,
                             freq_dim=freq_dim, attn_caches=caches[key], fp8=fp8, fp8_attention=fp8_attention)
        return f
    return euler_cfg_cached(noise, n_steps, guidance, vel(ctx_cond, "c"), vel(ctx_uncond, "u"), schedule)


# --------------------------------------------------------------------------------------
# FP8 (E4M3) linear layers  [Wan-P2, "Infra", inference optimisation: FP8 GEMM with a
# per-tensor scale for the weights and a per-token scale for the activations]
# --------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code: sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
    exponent field 0 holds the subnormals m/8 * 2^-6; there are no infinities and
    S.1111.111 is NaN."""
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def round_e4m3(x) -> np.ndarray:
    """Nearest E4M3 value (ties to the even code), saturated to +-448. Normal numbers
    (|x| >= 2^-6) have a spacing of 2^(e-3) in [2^e, 2^(e+1)); below 2^-6 the spacing is
    2^-9 (subnormals)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)
    q = np.exp2(e - 3)
    r = np.rint(a / q) * q                      # np.rint: round half to even
    r = np.minimum(r, E4M3_MAX)
    return np.sign(x) * r


def quantize_e4m3(x, axis=None):
    """Scale and codes for ``x ~ scale * q``: ``scale = amax / 448`` over the whole
    tensor (``axis=None``, weights) or per row (``axis=-1``, activations: one scale per
    token), ``q = round_e4m3(x / scale)``. reading: the scale maps the largest magnitude
    onto the largest code; an all-zero row or tensor gets scale 1. The scale and the
    division are float32 operations, the precision the kernels decide the code in.
    Returns ``(q, scale)`` with q as float64 values on the E4M3 grid."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=axis, keepdims=axis is not None).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = round_e4m3((x32 / scale).astype(np.float32))
    return q, (scale if axis is not None else np.float32(scale))


def linear_fp8(x, weight, bias=None) -> np.ndarray:
    """``y = (q_x q_w^T) * s_x[row] * s_w + b`` with per-token codes of the input and
    per-tensor codes of the weight (``quantize_e4m3``); the product of the codes is
    exact in float64."""
    qx, sx = quantize_e4m3(x, axis=-1)
    qw, sw = quantize_e4m3(weight)
    y = (qx @ qw.T) * sx.astype(np.float64) * np.float64(sw)
    return y if bias is None else y + _f(bias)


def attention_fp8(q, k, v, heads: int, running_base: bool = False, split_units=(), rows=None,
                  prob=None) -> np.ndarray:
    """8-bit attention [Wan-P2, "Infra", inference optimisation: 8-bit FlashAttention,
    INT8 for q k^T and FP8 for the product with v]. reading: E4M3 for both products (the
    8-bit format of the tensor cores' f8 kind), with these scales, each an amax / 448
    as in ``quantize_e4m3``:

    * q: one scale per (token, head) -- the per-token activation scale, per head since
      each head's q k^T is a separate product;
    * k and v: one scale per head over all key rows, so a key's scale does not vary
      along a row of the score matrix;
    * the probabilities, taken against a power-of-two base, ``p = 2^(x - ceil(max_j x))``
      with ``x`` the logit in log2 units (so the row's largest p lies in (1/2, 1]), are
      rounded to E4M3 without a further scale for the product with v; the normaliser
      is the sum of the unrounded p. (Softmax does not depend on the base; a power-of-
      two base makes the rounding of p the same for any base a whole power of two
      away, which a one-pass kernel with a running base can reproduce.)

    Per head: ``x = (q^ k^T) sq sk / (sqrt(d) ln 2)``, ``o = sv (E4M3(p) v^) / sum_j p``.

    ``running_base`` takes the base the way a one-pass kernel meets the keys instead of
    from the row's final maximum (``_running_base_rows``); the two agree exactly unless
    some p falls into E4M3's subnormal range under one base and not the other.
    ``split_units``: (head, query block) pairs whose keys a kernel took in two halves
    (query blocks of 256 rows). ``rows`` returns only those query rows (q still holds
    every row: under the running base a row's result depends on its 32-row group).
    ``prob`` (running base only): ``prob(S, c, base, first_key)`` evaluates a key tile's
    probabilities ``2^(S c - base)``; by default exactly, in float64. A caller may pass a
    model of some other arithmetic to study its effect."""
    q, k, v = (np.asarray(a, dtype=np.float32) for a in (q, k, v))
    Lq, D = q.shape
    d = D // heads
    sel = np.arange(Lq) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(sel), D), dtype=F64)
    for hh in range(heads):
        sl = slice(hh * d, (hh + 1) * d)
        kq, sk = quantize_e4m3(k[:, sl])
        vq, sv = quantize_e4m3(v[:, sl])
        if running_base:
            qq, sq = quantize_e4m3(q[:, sl], axis=-1)
            c = sq.astype(F64) * F64(sk) / (math.sqrt(d) * math.log(2.0))   # log2 units per unit of S
            split = {qb for (h2, qb) in split_units if h2 == hh}
            out[:, sl] = F64(sv) * _running_base_rows(qq, c, kq, vq, split, sel, prob=prob)
            continue
        qq, sq = quantize_e4m3(q[sel][:, sl], axis=-1)
        x = (qq @ kq.T) * sq.astype(F64) * F64(sk) / (math.sqrt(d) * math.log(2.0))
        p = np.exp2(x - np.ceil(x.max(axis=-1, keepdims=True)))
        out[:, sl] = F64(sv) * (round_e4m3(p) @ vq) / p.sum(axis=-1, keepdims=True)
    return out


def _running_base_rows(qq, c, kq, vq, split_blocks, rows, tile: int = 128, warp: int = 32, block: int = 256,
                       threshold: float = 8.0, prob=None) -> np.ndarray:
    """The rows ``rows`` of one head of ``attention_fp8`` with the base a one-pass kernel
    keeps. ``qq`` [Lq, d] and ``kq``, ``vq`` [Lk, d] are E4M3 values, ``c`` [Lq, 1] the
    log2 units of one unit of ``S = qq kq^T`` (exact). The keys come in tiles of ``tile``
    in order; a row's running maximum m of S starts at its first tile's maximum and
    moves to max(m, tile maximum) only when, for some row of its group of ``warp``
    consecutive rows (groups from row 0), the tile maximum exceeds m by more than
    ``threshold`` in log2 units -- then every row of the group moves; each tile's p is
    taken against ``ceil(m c)``, and what was summed before a move is scaled by the exact
    power of two between the old and the new base. Query blocks in ``split_blocks``
    (rows [256 b, 256 b + 256)) take their keys in two halves of the key tiles (the
    first floor(n/2) tiles, then the rest), each half with its own running base, merged
    as ``(w0 O0 + w1 O1) / (w0 l0 + w1 l1)`` with ``w_i = 2^(b_i - max(b0, b1))``.
    Returns the normalised ``E4M3(p) v^`` of those rows (without the v scale). ``prob``
    as in ``attention_fp8``."""
    Lq, Lk = qq.shape[0], kq.shape[0]
    if prob is None:
        def prob(St, cr, base, first_key):
            return np.exp2(St * cr - base)
    ntile = (Lk + tile - 1) // tile

    def one_pass(S, cr, t0, t1):
        # one group of rows over key tiles [t0, t1): (base, unnormalised output, sum)
        m = None
        o = np.zeros((S.shape[0], vq.shape[1]), dtype=F64)
        l = np.zeros((S.shape[0], 1), dtype=F64)
        for j in range(t0, t1):
            St = S[:, j * tile:min((j + 1) * tile, Lk)]
            mx = St.max(axis=-1, keepdims=True)
            if m is None:
                m = mx.copy()
            elif ((mx - m) * cr > threshold).any():
                m_new = np.maximum(m, mx)
                alpha = np.exp2(np.ceil(m * cr) - np.ceil(m_new * cr))
                o *= alpha
                l *= alpha
                m = m_new
            p = prob(St, cr, np.ceil(m * cr), j * tile)
            o += round_e4m3(p) @ vq[j * tile:j * tile + St.shape[1]]
            l += p.sum(axis=-1, keepdims=True)
        return np.ceil(m * cr), o, l

    out = np.empty((len(rows), vq.shape[1]), dtype=F64)
    where = {}
    for i, r in enumerate(rows):
        where.setdefault(int(r) // warp * warp, []).append(i)
    for w0, idx in where.items():
        w1 = min(w0 + warp, Lq)
        S, cr = qq[w0:w1] @ kq.T, c[w0:w1]
        if w0 // block in split_blocks:
            b0, o0, l0 = one_pass(S, cr, 0, ntile // 2)
            b1, o1, l1 = one_pass(S, cr, ntile // 2, ntile)
            bm = np.maximum(b0, b1)
            g0, g1 = np.exp2(b0 - bm), np.exp2(b1 - bm)
            res = (g0 * o0 + g1 * o1) / (g0 * l0 + g1 * l1)
        else:
            _, o, l = one_pass(S, cr, 0, ntile)
            res = o / l
        out[idx] = res[np.asarray(rows)[idx] - w0]
    return out


# --------------------------------------------------------------------------------------
# Full-size stack evaluation: float32 products, float64 reductions
# --------------------------------------------------------------------------------------
# The 30-block 1.3B stack at 480P (32760 tokens) is ~283 TFLOP; in float64 numpy it would
# take hours on a host. This variant computes the same definition (``dit_stack``, the
# flow-matching input of [Wan-P2, "训练方法"]) with every matrix product in float32 (the
# products of float32 numbers accumulate in float32 inside the BLAS) and everything else
# in float64: the residual stream, LayerNorm (mean and variance), modulation, GELU,
# biases, the softmax row maximum and the row sum. The softmax exponentials are float32
# values of the float32 logits. Its distance from the float64 definition (~1e-6 relative)
# is pinned against ``dit_stack`` at small sizes. torch's CPU ops serve as the library
# steps (multi-threaded matmul, exp and sum), nothing else.

def _t32(a):
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(torch.float32).contiguous()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def _t64(a):
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(torch.float64)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def linear_f32(x, weight, bias=None):
    """``x W^T`` as a float32 product, plus the bias in float64; returns float64."""
    import torch
    y = (_t32(x) @ _t32(weight).T).to(torch.float64)
    return y if bias is None else y + _t64(bias)


def layer_norm_f64(x, eps: float = 1e-6):
    """``layer_norm`` on a torch float64 tensor (same definition)."""
    x = _t64(x)
    mu = x.mean(dim=-1, keepdim=True)
    var = ((x - mu) ** 2).mean(dim=-1, keepdim=True)
    return (x - mu) / (var + eps).sqrt()


def attention_f32(q, k, v, heads: int, chunk: int = 2048):
    """``attention`` with the two products in float32: per head and per block of query
    rows, ``s = q k^T`` (float32), ``p = exp((s - max_j s) / sqrt(d))`` (float32
    exponentials), ``l = sum_j p`` (float64 over float32 partial sums of 128
    consecutive keys), ``o = (p v) / l`` (the product in float32)."""
    import torch
    q32, k32, v32 = _t32(q), _t32(k), _t32(v)
    Lq, D = q32.shape
    Lk = k32.shape[0]
    d = D // heads
    nb = Lk // 128
    out = torch.empty((Lq, D), dtype=torch.float64)
    buf = torch.empty((min(chunk, Lq), Lk), dtype=torch.float32)
    for hh in range(heads):
        sl = slice(hh * d, (hh + 1) * d)
        khT, vh = k32[:, sl].T.contiguous(), v32[:, sl].contiguous()
        for r0 in range(0, Lq, chunk):
            qc = q32[r0:r0 + chunk, sl]
            s = buf[:qc.shape[0]]
            torch.matmul(qc, khT, out=s)
            s.sub_(s.amax(dim=-1, keepdim=True)).mul_(1.0 / math.sqrt(d)).exp_()
            l = s[:, :nb * 128].reshape(s.shape[0], nb, 128).sum(dim=-1).to(torch.float64).sum(dim=-1, keepdim=True)
            l += s[:, nb * 128:].sum(dim=-1, keepdim=True).to(torch.float64)
            out[r0:r0 + chunk, sl] = (s @ vh).to(torch.float64) / l
    return out


def ffn_f32(h, w: Dict[str, np.ndarray], chunk: int = 4096):
    """``ffn_branch`` with float32 products; the hidden layer (bias, GELU-tanh) in
    float64, a block of rows at a time (rows are independent)."""
    import torch
    h = _t64(h)
    out = torch.empty((h.shape[0], _f(w["w_2"]).shape[0]), dtype=torch.float64)
    for r0 in range(0, h.shape[0], chunk):
        u = linear_f32(h[r0:r0 + chunk], w["w_1"], w["b_1"])
        u = 0.5 * u * (1.0 + torch.tanh(math.sqrt(2.0 / math.pi) * (u + 0.044715 * u ** 3)))
        out[r0:r0 + chunk] = linear_f32(u, w["w_2"], w["b_2"])
    return out


def dit_block_f32(x, e, w: Dict[str, np.ndarray], ctx, heads: int, eps: float = 1e-6, img_ctx=None,
                  rows: Optional[Sequence[int]] = None):
    """``dit_block`` with float32 products and float64 reductions (the section comment
    above). ``x`` and the result are float64 torch tensors; ``rows`` as in ``dit_block``."""
    import torch
    x = _t64(x)
    D = x.shape[-1]
    shift_msa, scale_msa, gate_msa, shift_ffn, scale_ffn, gate_ffn = _t64(block_modulation(e, w["mod_bias"]))
    h_all = layer_norm_f64(x, eps) * (1.0 + scale_msa) + shift_msa
    if rows is None:
        xr, hr = x, h_all
    else:
        idx = torch.from_numpy(np.asarray(rows, dtype=np.int64))
        xr, hr = x[idx], h_all[idx]
    wqkv, bqkv = w["w_qkv"], _f(w["b_qkv"])
    q = linear_f32(hr, wqkv[:D], bqkv[:D])
    kv = linear_f32(h_all, wqkv[D:], bqkv[D:])
    o = attention_f32(q, kv[:, :D], kv[:, D:], heads)
    x1 = xr + gate_msa * linear_f32(o, w["w_o"], w["b_o"])
    hc = layer_norm_f64(x1, eps)
    qc = linear_f32(hc, w["w_cq"], w["b_cq"])
    kvc = linear_f32(ctx, w["w_ckv"], w["b_ckv"])
    oc = attention_f32(qc, kvc[:, :D], kvc[:, D:], heads)
    if img_ctx is not None:
        kvi = linear_f32(img_ctx, w["w_ckv_img"], w["b_ckv_img"])
        oc = oc + attention_f32(qc, kvi[:, :D], kvi[:, D:], heads)
    x2 = x1 + linear_f32(oc, w["w_co"], w["b_co"])
    hf = layer_norm_f64(x2, eps) * (1.0 + scale_ffn) + shift_ffn
    return x2 + gate_ffn * ffn_f32(hf, w)


def dit_stack_f32(latent, t: float, weights: Dict, blocks: Sequence[Dict], ctx, heads: int,
                  eps: float = 1e-6, img_ctx=None, freq_dim: int = 256,
                  rows: Optional[Sequence[int]] = None, progress=None) -> np.ndarray:
    """``dit_stack`` with the blocks and the head in float32 products and float64
    reductions (patchify and the time MLP are the float64 functions above). With
    ``rows`` the last block and the head are evaluated for those tokens only (every
    earlier block needs all tokens) and the result is the head output ``[len(rows),
    out_ch*4]``; otherwise it is the unpatchified velocity ``[out_ch, F, H, W]``.
    ``progress(i)`` is called after block ``i``."""
    lat = _f(latent)
    C, F, H, W = lat.shape
    x = _t64(patchify(lat, weights["w_p"], weights["b_p"]))
    e = time_mlp(t, weights["w_t1"], weights["b_t1"], weights["w_t2"], weights["b_t2"], freq_dim)
    n = len(blocks)
    for i, blk in enumerate(blocks):
        x = dit_block_f32(x, e, blk, ctx, heads, eps, img_ctx=img_ctx,
                          rows=rows if i == n - 1 else None)
        if progress is not None:
            progress(i)
    if rows is not None and n == 0:
        x = x[_t64(np.asarray(rows)).long()]
    y = linear_f32(layer_norm_f64(x, eps), weights["w_head"], weights["b_head"]).numpy()
    if rows is not None:
        return y
    return unpatchify(y, _f(weights["w_head"]).shape[0] // 4, F, H, W)
