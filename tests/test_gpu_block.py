"""Block- and stack-level parity of the C ABI with the CPU oracle at sizes the oracle
finishes in seconds: the tiny fp32 workload on all rows, reduced-width bf16 blocks
(T2V and I2V) spanning several tiles with ragged tails, and a short stack."""
import dataclasses

import numpy as np
import pytest

from oracle import wan_oracle as O
from wan_inputs import WORKLOADS, make_inputs
from gpu_util import BF16_TOL, F32_TOL, host, rel_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wan():
    import video_diffusion_transformer_wan_b200 as w
    return w


def small_bf16(i2v=False, **kw):
    base = WORKLOADS["wan13b_480p_i2v_block" if i2v else "wan13b_480p_block"]
    d = dict(frames=3, height=10, width=14, dim=256, heads=2, ffn=512, text_len=40)
    if i2v:
        d.update(img_len=7, img_feat=64)
    d.update(kw)
    return dataclasses.replace(base, **d)


class Run:
    """Inputs on the device and the ABI tables for one workload."""

    def __init__(self, wan, w, seed=0, n_blocks=None, zero_wx=True, uncond=False):
        from video_diffusion_transformer_wan_b200.model import DitModel, config_for, to_device
        self.w = w
        self.inp = make_inputs(w, seed=seed, n_blocks=n_blocks, zero_wx=zero_wx, uncond=uncond)
        self.cfg = config_for(w)
        self.model = DitModel(self.cfg, self.inp)
        act = self.model.act
        self.act = act
        self.x = to_device(self.inp["x"], torch.float32)
        self.e = to_device(self.inp["e"], torch.float32)
        self.ctx = to_device(self.inp["ctx"], act)
        self.ctx_uncond = to_device(self.inp["ctx_uncond"], act) if uncond else None
        self.img_ctx = None
        self.img_np = None
        Li = 0
        if w.i2v:
            Li = w.img_len
            feat = to_device(self.inp["img_feat"], act)
            self.img_ctx = torch.empty(w.batch, Li, w.dim, dtype=act, device="cuda")
            ws = torch.empty(2 * w.batch * Li * w.dim * 4, dtype=torch.uint8, device="cuda")
            wan.image_context_fwd(self.cfg, feat, self.model.image_table, self.img_ctx, ws)
            self.img_np = [O.image_context_mlp(self.inp["img_feat"][b], *(self.inp[k] for k in
                           ["w_i1", "b_i1", "w_i2", "b_i2", "w_i3", "b_i3"])) for b in range(w.batch)]
        self.ws = torch.empty(wan.workspace_bytes(self.cfg, w.batch, w.tokens, w.text_len, Li), dtype=torch.uint8,
                              device="cuda")


@pytest.mark.parametrize("name", ["tiny_f32_block", "small_bf16", "small_bf16_i2v", "small_bf16_b2"])
def test_block_matches_oracle_all_rows(wan, name):
    if name == "tiny_f32_block":
        w = WORKLOADS[name]
    elif name == "small_bf16":
        w = small_bf16()
    elif name == "small_bf16_i2v":
        w = small_bf16(i2v=True)
    else:
        w = small_bf16(batch=2, frames=2, height=12, width=22)
    r = Run(wan, w)
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    x0 = host(r.x)
    xg = r.x.clone()
    wan.dit_block_fwd(r.cfg, xg, r.e, r.ctx, r.img_ctx, r.model.block_tables[0], r.ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(xg)
    blk = r.inp["blocks"][0]
    for b in range(w.batch):
        img = None if r.img_np is None else r.img_np[b]
        ref, parts = O.dit_block(r.inp["x"][b], r.inp["e"][b], blk, r.inp["ctx"][b], w.heads, img_ctx=img,
                                 return_parts=True)
        assert rel_err(got[b], ref) <= tol
        assert rel_err(got[b] - x0[b], ref - x0[b]) <= tol, "branch delta"
        if r.img_np is not None:
            # the image context itself
            assert rel_err(host(r.img_ctx)[b], img) <= BF16_TOL


@pytest.mark.parametrize("name", ["tiny_f32_block", "small_bf16", "small_bf16_i2v"])
def test_branch_calls_match_oracle(wan, name):
    """Each sub-call's own delta is checked, so a wrong branch cannot hide behind the
    residual stream."""
    w = WORKLOADS[name] if name == "tiny_f32_block" else small_bf16(i2v=name.endswith("i2v"))
    r = Run(wan, w)
    tol = F32_TOL if w.dtype == "f32" else BF16_TOL
    blk = r.inp["blocks"][0]
    bw = r.model.block_tables[0]
    mb = r.model.blocks[0]["mod_bias"]
    B, L, D = w.batch, w.tokens, w.dim
    h = torch.empty(B, L, D, dtype=r.act, device="cuda")
    x = r.x.clone()
    # self-attention branch
    wan.adaln_modulate(r.cfg, x, r.e, mb, 0, h)
    wan.self_attn_fwd(r.cfg, h, bw, r.e, x, r.ws)
    torch.cuda.synchronize()
    x1 = host(x)
    for b in range(B):
        mod = O.block_modulation(r.inp["e"][b], blk["mod_bias"])
        hm = O.modulate(O.layer_norm(r.inp["x"][b]), mod[0], mod[1])
        assert rel_err(host(h)[b], hm) <= tol
        sa = O.self_attention_branch(hm, blk, w.heads)
        assert rel_err(x1[b] - r.inp["x"][b], mod[2] * sa) <= tol
    # cross-attention branch (from the GPU state x1, compared with the oracle on x1)
    wan.adaln_modulate(r.cfg, x, None, None, -1, h)
    wan.cross_attn_fwd(r.cfg, h, r.ctx, r.img_ctx, bw, x, r.ws)
    torch.cuda.synchronize()
    x2 = host(x)
    for b in range(B):
        hc = O.layer_norm(x1[b])
        img = None if r.img_np is None else r.img_np[b]
        ca = O.cross_attention_branch(hc, r.inp["ctx"][b], blk, w.heads, img_ctx=img)
        assert rel_err(x2[b] - x1[b], ca) <= tol
    # FFN branch
    wan.adaln_modulate(r.cfg, x, r.e, mb, 1, h)
    wan.ffn_fwd(r.cfg, h, bw, r.e, x, r.ws)
    torch.cuda.synchronize()
    x3 = host(x)
    for b in range(B):
        mod = O.block_modulation(r.inp["e"][b], blk["mod_bias"])
        hf = O.modulate(O.layer_norm(x2[b]), mod[3], mod[4])
        assert rel_err(x3[b] - x2[b], mod[5] * O.ffn_branch(hf, blk)) <= tol


def test_zero_gates_and_identity_block(wan):
    """Zero gates leave only the cross-attention delta; zeroing its output projection
    too makes the block the identity, exactly, on the GPU."""
    w = small_bf16()
    r = Run(wan, w)
    mb = r.model.blocks[0]["mod_bias"]
    e0 = r.e.clone()
    e0[:, 2] = -mb[2]
    e0[:, 5] = -mb[5]
    blk = dict(r.model.blocks[0])
    blk["w_co"] = torch.zeros_like(blk["w_co"])
    blk["b_co"] = torch.zeros_like(blk["b_co"])
    bw = wan.block_weights(blk)
    x = r.x.clone()
    wan.dit_block_fwd(r.cfg, x, e0, r.ctx, None, bw, r.ws)
    torch.cuda.synchronize()
    assert torch.equal(x, r.x)


def test_block_repeatable_and_text_permutation(wan):
    w = small_bf16()
    r = Run(wan, w)
    x1, x2 = r.x.clone(), r.x.clone()
    bw = r.model.block_tables[0]
    wan.dit_block_fwd(r.cfg, x1, r.e, r.ctx, None, bw, r.ws)
    wan.dit_block_fwd(r.cfg, x2, r.e, r.ctx, None, bw, r.ws)
    perm = torch.randperm(w.text_len, generator=torch.Generator().manual_seed(0)).cuda()
    x3 = r.x.clone()
    wan.dit_block_fwd(r.cfg, x3, r.e, r.ctx[:, perm].contiguous(), None, bw, r.ws)
    torch.cuda.synchronize()
    assert torch.equal(x1, x2)                       # bitwise deterministic
    d = (x3 - r.x).abs().max() / (x1 - r.x).abs().max()
    assert rel_err(host(x3 - r.x), host(x1 - r.x)) <= 5e-3, float(d)


@pytest.mark.parametrize("i2v", [False, True])
def test_stack_matches_oracle(wan, i2v):
    """Patchify, the shared timestep MLP with per-block biases, two blocks, the head and
    unpatchify; for I2V the 36-channel input is built on the GPU from the frame mask."""
    w = small_bf16(i2v=i2v, n_blocks=2)
    r = Run(wan, w, zero_wx=False)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    t = torch.from_numpy(r.inp["t"]).cuda()
    noise = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    if i2v:
        cond = torch.from_numpy(r.inp["cond"]).cuda().to(r.act)
        keep = np.zeros((B, 1 + 4 * (F - 1)), np.uint8)
        keep[:, 0] = 1
        lat = torch.empty(B, 36, F, H, W, dtype=r.act, device="cuda")
        wan.i2v_input(r.cfg, noise, cond, torch.from_numpy(keep).cuda(), lat)
    else:
        lat = noise
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(r.cfg, lat, t, r.model.stack_table, r.model.block_tables, r.ctx, r.img_ctx, v, r.ws)
    torch.cuda.synchronize()
    got = host(v)
    for b in range(B):
        if i2v:
            lat_np = O.i2v_input(r.inp["noise"][b], r.inp["cond"][b], O.i2v_mask(keep[b], F, H, W))
        else:
            lat_np = r.inp["noise"][b]
        ref = O.dit_stack(lat_np, float(r.inp["t"][b]), r.inp, r.inp["blocks"], r.inp["ctx"][b], w.heads,
                          img_ctx=None if r.img_np is None else r.img_np[b])
        assert rel_err(got[b], ref) <= BF16_TOL


def test_stack_equals_patchify_blocks_head(wan):
    """The stack call equals its parts called one by one through the ABI, bitwise."""
    w = small_bf16(n_blocks=2)
    r = Run(wan, w)
    B, F, H, W, D, L = w.batch, w.frames, w.height, w.width, w.dim, w.tokens
    lat = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    t = torch.from_numpy(r.inp["t"]).cuda()
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(r.cfg, lat, t, r.model.stack_table, r.model.block_tables, r.ctx, None, v, r.ws)
    x = torch.empty(B, L, D, dtype=torch.float32, device="cuda")
    ws2 = torch.empty_like(r.ws)
    s = r.model.stack
    wan.patchify(r.cfg, lat, s["w_p"], s["b_p"], x, ws2)
    e = torch.empty(B, 6, D, dtype=torch.float32, device="cuda")
    wan.time_mlp(r.cfg, t, r.model.time_table, e)
    for bw in r.model.block_tables:
        wan.dit_block_fwd(r.cfg, x, e, r.ctx, None, bw, ws2)
    v2 = torch.empty_like(v)
    wan.head_fwd(r.cfg, x, F, H, W, s["w_head"], s["b_head"], v2, ws2)
    torch.cuda.synchronize()
    assert torch.equal(v, v2)


def test_flow_matching_velocity_and_loss(wan):
    """One rectified-flow velocity evaluation: x_t = u x1 + (1-u) x0 and t = 1000 u on the
    GPU, the stack's prediction, and the MSE against x1 - x0."""
    w = small_bf16(n_blocks=1, flow_matching=True)
    r = Run(wan, w)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    x1 = torch.from_numpy(r.inp["x1"]).cuda().to(r.act)
    x0 = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    u = torch.from_numpy(r.inp["u"]).cuda()
    xt = torch.empty_like(x1)
    t = torch.empty(B, dtype=torch.float32, device="cuda")
    wan.flow_matching_input(r.cfg, x1, x0, u, xt, t)
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(r.cfg, xt, t, r.model.stack_table, r.model.block_tables, r.ctx, None, v, r.ws)
    loss = torch.empty(B, dtype=torch.float32, device="cuda")
    wan.flow_matching_loss(r.cfg, v, x1, x0, loss)
    torch.cuda.synchronize()
    for b in range(B):
        xt_ref = O.flow_matching_input(r.inp["x1"][b], r.inp["noise"][b], float(r.inp["u"][b]))
        ref = O.dit_stack(xt_ref, 1000.0 * float(r.inp["u"][b]), r.inp, r.inp["blocks"],
                          r.inp["ctx"][b], w.heads)
        assert rel_err(host(v)[b], ref) <= BF16_TOL
        ref_loss = np.mean((ref - O.flow_matching_target(r.inp["x1"][b], r.inp["noise"][b])) ** 2)
        assert abs(float(loss[b]) - ref_loss) / ref_loss < 1e-2


@pytest.mark.parametrize("frames,height,width,text_len,batch", [(5, 40, 44, 300, 2), (5, 40, 42, 40, 1)])
def test_block_with_key_split_tail(wan, frames, height, width, text_len, batch):
    """Few work units (fewer than half the SMs), so every self-attention unit is split
    over its key tiles (18 and 17 of them, L = 2200 and 2100) and the halves are merged;
    all rows against the oracle."""
    w = small_bf16(frames=frames, height=height, width=width, text_len=text_len, batch=batch)
    r = Run(wan, w, zero_wx=False)
    x = r.x.clone()
    wan.dit_block_fwd(r.cfg, x, r.e, r.ctx, None, r.model.block_tables[0], r.ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(x)
    for b in range(w.batch):
        ref = O.dit_block(r.inp["x"][b], r.inp["e"][b], r.inp["blocks"][0], r.inp["ctx"][b], w.heads)
        assert rel_err(got[b] - r.inp["x"][b], ref - r.inp["x"][b]) <= BF16_TOL
