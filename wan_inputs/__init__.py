"""Seeded synthetic inputs for the Wan 2.1 DiT hot path.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It only draws random numbers and converts dtypes; it holds none of
the method's arithmetic (no normalisation, projection, attention or embedding).

Workloads follow the model table of "Wan: Open and Advanced Large-Scale Video
Generative Models (Wan 2.1)" (zhao9797.github.io, section "Diffusion
Transformer", config table): 1.3B = dim 1536, FFN 8960, 12 heads, 30 layers;
14B = dim 5120, FFN 13824, 40 heads, 40 layers; latent in/out dim 16, frequency
dim 256, 512 text tokens (section "umT5").

Distributions: every weight and bias ~ N(0, 0.02); latents, text context and
image features ~ N(0, 1); timestep t ~ U(0, 1000) (block-level workloads) or
flow-matching t ~ U(0, 1) scaled by 1000 (stack workload). Draws come from
numpy ``Generator(PCG64(seed))`` in the fixed order listed in ``make_inputs``.
Values meant to be stored in bf16 are rounded to bf16 (round to nearest even)
here, once, so both the CUDA path and the oracle read identical numbers.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "make_inputs", "round_bf16", "bf16_bits",
    "bits_to_f32", "sample_rows", "block_weight_names", "input_digest",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": storage/compute type of weights and activations
    batch: int
    in_ch: int            # DiT input channels (16 for T2V, 36 for I2V)
    frames: int           # latent frames  = 1 + T/4
    height: int           # latent height  = H_pixels / 8
    width: int            # latent width   = W_pixels / 8
    dim: int
    heads: int
    ffn: int
    text_len: int
    img_len: int = 0      # image-context tokens (I2V only)
    img_feat: int = 1280  # image-encoder feature width (I2V only)
    n_blocks: int = 1
    out_ch: int = 16
    freq_dim: int = 256
    eps: float = 1e-6
    flow_matching: bool = False

    @property
    def head_dim(self) -> int:
        return self.dim // self.heads

    @property
    def tokens(self) -> int:
        # (1,2,2) patches over the latent grid: frames * (H/2) * (W/2)
        return self.frames * (self.height // 2) * (self.width // 2)

    @property
    def i2v(self) -> bool:
        return self.img_len > 0


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 block: latent 16x2x8x8 -> 32 tokens, dim 128, 2 heads, FFN 512, 16 text tokens
    "tiny_f32_block": Workload("tiny_f32_block", "f32", 1, 16, 2, 8, 8, 128, 2, 512, 16),
    # Wan 1.3B block at 480P, 81 frames: latent 16x21x60x104 -> 32760 tokens
    "wan13b_480p_block": Workload("wan13b_480p_block", "bf16", 1, 16, 21, 60, 104, 1536, 12, 8960, 512),
    # Wan 1.3B full 30-block stack with one flow-matching velocity evaluation
    "wan13b_480p_stack30": Workload("wan13b_480p_stack30", "bf16", 1, 16, 21, 60, 104, 1536, 12, 8960, 512,
                                    n_blocks=30, flow_matching=True),
    # Wan 14B block at 720P, 81 frames: latent 16x21x90x160 -> 75600 tokens
    "wan14b_720p_block": Workload("wan14b_720p_block", "bf16", 1, 16, 21, 90, 160, 5120, 40, 13824, 512),
    # I2V at the 1.3B shape: 16 noise + 16 condition + 4 mask channels, 257 image tokens
    "wan13b_480p_i2v_block": Workload("wan13b_480p_i2v_block", "bf16", 1, 36, 21, 60, 104, 1536, 12, 8960, 512,
                                      img_len=257),
}


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bf16 (ties to even); returns float32."""
    return bits_to_f32(bf16_bits(a))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of float values, round to nearest even."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def block_weight_names(w: Workload) -> List[str]:
    names = ["mod_bias", "w_qkv", "b_qkv", "w_o", "b_o", "w_cq", "b_cq", "w_ckv", "b_ckv", "w_co", "b_co"]
    if w.i2v:
        names += ["w_ckv_img", "b_ckv_img"]
    names += ["w_1", "b_1", "w_2", "b_2"]
    return names


def _block_shapes(w: Workload) -> Dict[str, tuple]:
    D, F = w.dim, w.ffn
    return {
        "mod_bias": (6, D),
        "w_qkv": (3 * D, D), "b_qkv": (3 * D,),
        "w_o": (D, D), "b_o": (D,),
        "w_cq": (D, D), "b_cq": (D,),
        "w_ckv": (2 * D, D), "b_ckv": (2 * D,),
        "w_co": (D, D), "b_co": (D,),
        "w_ckv_img": (2 * D, D), "b_ckv_img": (2 * D,),
        "w_1": (F, D), "b_1": (F,),
        "w_2": (D, F), "b_2": (D,),
    }


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def make_inputs(w: Workload, seed: int = 0, *, n_blocks: Optional[int] = None,
                zero_wx: bool = True, block_input: bool = True, uncond: bool = False) -> Dict[str, object]:
    """Draw every tensor of a workload, in this fixed order:

    1. latent noise ``[B,16,F,H,W]`` ~ N(0,1)
    2. (I2V) condition latent ``[B,16,F,H,W]`` ~ N(0,1)
    3. text context ``[B,Lc,D]`` ~ N(0,1)
    4. (I2V) image features ``[B,Li,1280]`` ~ N(0,1)
    5. timestep: ``t [B]`` ~ U(0,1000); for flow matching ``u [B]`` ~ U(0,1) and
       a second latent x1 ``[B,16,F,H,W]`` ~ N(0,1) (the noise above is x0)
    6. patchify weight ``[D,Cin,1,2,2]`` and bias ``[D]``; for I2V the last 20 input
       channels' slice of the weight is zero when ``zero_wx`` (zero-initialised extra
       projection) and N(0,0.02) otherwise
    7. time MLP: ``w_t1 [D,256]``, ``b_t1 [D]``, ``w_t2 [6D,D]``, ``b_t2 [6D]``
    8. (I2V) image MLP: ``w_i1 [D,1280]``, ``b_i1``, ``w_i2 [D,D]``, ``b_i2``, ``w_i3 [D,D]``, ``b_i3``
    9. per block, in ``block_weight_names`` order (``mod_bias`` [6,D] fp32)
    10. head: ``w_head [64,D]``, ``b_head [64]``
    11. (block_input) a residual-stream block input ``x [B,L,D]`` ~ N(0,1) fp32 and a
        shared-MLP output ``e [B,6,D]`` ~ N(0,0.2) fp32, for the block-level sub-calls.
    12. (uncond) a second text context ``ctx_uncond [B,Lc,D]`` ~ N(0,1), the
        unconditional branch of guided sampling (drawn last so that it leaves every
        other tensor of the seed unchanged).

    Weights and biases (except ``mod_bias``), latents, context and image features are
    rounded to bf16 for bf16 workloads; everything stays fp32 for f32 workloads.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    B, D, L = w.batch, w.dim, w.tokens
    nb = w.n_blocks if n_blocks is None else n_blocks
    rb = round_bf16 if w.dtype == "bf16" else (lambda a: a.astype(np.float32))
    lat_shape = (B, 16, w.frames, w.height, w.width)
    out: Dict[str, object] = {"workload": w, "seed": seed}

    out["noise"] = rb(_normal(rng, lat_shape, 1.0))
    if w.i2v:
        out["cond"] = rb(_normal(rng, lat_shape, 1.0))
    out["ctx"] = rb(_normal(rng, (B, w.text_len, D), 1.0))
    if w.i2v:
        out["img_feat"] = rb(_normal(rng, (B, w.img_len, w.img_feat), 1.0))
    if w.flow_matching:
        out["u"] = rng.uniform(0.0, 1.0, size=(B,)).astype(np.float32)
        out["x1"] = rb(_normal(rng, lat_shape, 1.0))
    else:
        out["t"] = rng.uniform(0.0, 1000.0, size=(B,)).astype(np.float32)

    wp = _normal(rng, (D, w.in_ch, 1, 2, 2), 0.02)
    if w.i2v and zero_wx:
        wp[:, 16:] = 0.0
    out["w_p"] = rb(wp)
    out["b_p"] = rb(_normal(rng, (D,), 0.02))

    out["w_t1"] = rb(_normal(rng, (D, w.freq_dim), 0.02))
    out["b_t1"] = rb(_normal(rng, (D,), 0.02))
    out["w_t2"] = rb(_normal(rng, (6 * D, D), 0.02))
    out["b_t2"] = rb(_normal(rng, (6 * D,), 0.02))

    if w.i2v:
        out["w_i1"] = rb(_normal(rng, (D, w.img_feat), 0.02))
        out["b_i1"] = rb(_normal(rng, (D,), 0.02))
        out["w_i2"] = rb(_normal(rng, (D, D), 0.02))
        out["b_i2"] = rb(_normal(rng, (D,), 0.02))
        out["w_i3"] = rb(_normal(rng, (D, D), 0.02))
        out["b_i3"] = rb(_normal(rng, (D,), 0.02))

    shapes = _block_shapes(w)
    blocks = []
    for _ in range(nb):
        blk = {}
        for name in block_weight_names(w):
            a = _normal(rng, shapes[name], 0.02)
            blk[name] = a if name == "mod_bias" else rb(a)
        blocks.append(blk)
    out["blocks"] = blocks

    out["w_head"] = rb(_normal(rng, (w.out_ch * 4, D), 0.02))
    out["b_head"] = rb(_normal(rng, (w.out_ch * 4,), 0.02))

    if block_input:
        out["x"] = _normal(rng, (B, L, D), 1.0)
        out["e"] = _normal(rng, (B, 6, D), 0.2)
    if uncond:
        out["ctx_uncond"] = rb(_normal(rng, (B, w.text_len, D), 1.0))
    return out


def sample_rows(n_rows: int, tile: int = 128, count: int = 256, seed: int = 0) -> np.ndarray:
    """Query rows checked at long sequence lengths: row 0, row n-1, every row of the
    ragged last tile, then seeded random rows up to ``count``; sorted, unique."""
    if n_rows <= count:
        return np.arange(n_rows)
    rows = {0, n_rows - 1}
    tail = n_rows % tile
    rows.update(range(n_rows - tail, n_rows))
    rng = np.random.Generator(np.random.PCG64(seed))
    while len(rows) < count:
        rows.add(int(rng.integers(0, n_rows)))
    return np.array(sorted(rows), dtype=np.int64)


def input_digest(inp: Dict[str, object]) -> str:
    """SHA-256 over every array of a ``make_inputs`` result (keys in sorted order, block
    dicts in block order, each array's dtype, shape and bytes). A stored expected value
    records it, so a change of the input recipe shows up as a digest mismatch rather
    than as a numerical failure."""
    h = hashlib.sha256()

    def add(name, a):
        a = np.ascontiguousarray(a)
        h.update(f"{name}:{a.dtype.str}:{a.shape};".encode())
        h.update(a.view(np.uint8).reshape(-1).data)

    for key in sorted(inp):
        val = inp[key]
        if isinstance(val, np.ndarray):
            add(key, val)
        elif key == "blocks":
            for i, blk in enumerate(val):
                for name in sorted(blk):
                    add(f"blocks[{i}].{name}", blk[name])
    return h.hexdigest()
