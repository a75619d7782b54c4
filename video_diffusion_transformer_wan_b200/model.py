"""Device-resident Wan 2.1 DiT weights and the ABI weight tables that point at them.

Marshalling only: host arrays are copied to the GPU once and the C structs
(``BlockWeights``, ``StackWeights``, ...) are filled with their device pointers.
Array names follow ``include/wan.h``: per block ``mod_bias, w_qkv, b_qkv, w_o, b_o,
w_cq, b_cq, w_ckv, b_ckv, w_co, b_co, [w_ckv_img, b_ckv_img,] w_1, b_1, w_2, b_2``;
stack ``w_p, b_p, w_t1, b_t1, w_t2, b_t2, w_head, b_head``; I2V image MLP
``w_i1, b_i1, w_i2, b_i2, w_i3, b_i3``.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np
import torch

from . import (BlockWeights, Config, Fp8Scales, ImageMlpWeights, StackWeights, TimeWeights, block_weights,
               fp8_quantize_tensor, make_config)


def to_device(a, dtype: torch.dtype, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device=device).to(dtype).contiguous()


class DitModel:
    """Weights of a DiT (any number of blocks) resident in device memory."""

    def __init__(self, cfg: Config, host: Dict[str, object], device="cuda"):
        self.cfg = cfg
        self.act = torch.bfloat16 if cfg.dtype == 1 else torch.float32
        up = lambda a: to_device(a, self.act, device)  # noqa: E731
        self.blocks: List[Dict[str, torch.Tensor]] = []
        for b in host.get("blocks", []):
            d = {k: (to_device(v, torch.float32, device) if k == "mod_bias" else up(v)) for k, v in b.items()}
            self.blocks.append(d)
        self.block_tables = [block_weights(b) for b in self.blocks]
        self.stack = {}
        for k in ["w_p", "b_p", "w_t1", "b_t1", "w_t2", "b_t2", "w_head", "b_head",
                  "w_i1", "b_i1", "w_i2", "b_i2", "w_i3", "b_i3"]:
            if k in host:
                a = np.asarray(host[k])
                if k == "w_p":
                    a = a.reshape(a.shape[0], -1)
                self.stack[k] = up(a)
        s = self.stack
        self.time_table = TimeWeights(*(s[k].data_ptr() if k in s else None for k in ["w_t1", "b_t1", "w_t2", "b_t2"]))
        self.stack_table = StackWeights(
            s["w_p"].data_ptr() if "w_p" in s else None, s["b_p"].data_ptr() if "b_p" in s else None,
            self.time_table, s["w_head"].data_ptr() if "w_head" in s else None,
            s["b_head"].data_ptr() if "b_head" in s else None)
        self.image_table: Optional[ImageMlpWeights] = None
        if "w_i1" in s:
            self.image_table = ImageMlpWeights(*(s[k].data_ptr() for k in ["w_i1", "b_i1", "w_i2", "b_i2",
                                                                           "w_i3", "b_i3"]))


def config_for(workload) -> Config:
    """ABI config of a ``wan_inputs.Workload``-like object."""
    return make_config(workload.dim, workload.heads, workload.ffn, in_ch=workload.in_ch, out_ch=workload.out_ch,
                       freq_dim=workload.freq_dim, img_feat=workload.img_feat, eps=workload.eps,
                       dtype=workload.dtype)


FP8_WEIGHTS = {"w_qkv": "qkv", "w_o": "o", "w_cq": "cq", "w_ckv": "ckv", "w_co": "co", "w_ckv_img": "ckv_img",
               "w_1": "ffn1", "w_2": "ffn2"}


class Fp8Block:
    """A block's weights as E4M3 codes with per-tensor scales, quantised on the GPU by
    ``wan_fp8_quantize_tensor`` from the bf16 device weights; biases and ``mod_bias``
    are shared with the bf16 block. ``attention_fp8``: the block's self-attention runs on
    E4M3 operands too."""

    def __init__(self, cfg: Config, block: Dict[str, torch.Tensor], attention_fp8: bool = False):
        self.codes: Dict[str, torch.Tensor] = {}
        self.scales: Dict[str, torch.Tensor] = {}
        for name, key in FP8_WEIGHTS.items():
            if name not in block:
                continue
            w = block[name]
            q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
            sc = torch.empty(1, dtype=torch.float32, device=w.device)
            fp8_quantize_tensor(cfg, w, q, sc)
            self.codes[name], self.scales[key] = q, sc
        tables = dict(block)
        tables.update(self.codes)
        self.table = block_weights(tables)
        self.scale_table = Fp8Scales(*(self.scales[k].data_ptr() if k in self.scales else None
                                       for k in ["qkv", "o", "cq", "ckv", "co", "ckv_img", "ffn1", "ffn2"]),
                                     1 if attention_fp8 else 0)
