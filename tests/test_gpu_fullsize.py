"""Parity at the full workload sizes, in the launch configuration bench.py times
(``wan_dit_stack_fwd``): 256 sampled query rows (rows 0 and L-1 and the whole ragged
last tile included) are compared with the oracle, which evaluates exactly those rows
(keys and values over all rows). Everything but self-attention is row-local, so this
is exact. The 30-block stack is checked at full size against the oracle's velocity of
256 sampled tokens (stored by a committed script that calls only the oracle), at
reduced token count with full-width blocks, and at full size through properties that
hold at any size."""
import dataclasses
import os

import numpy as np
import pytest

from oracle import wan_oracle as O
from wan_inputs import WORKLOADS, input_digest, make_inputs, sample_rows
from gpu_util import BF16_TOL, rel_err, rms_err

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wan():
    import video_diffusion_transformer_wan_b200 as w
    return w


def _setup(wan, w, inp):
    from video_diffusion_transformer_wan_b200.model import DitModel, config_for, to_device
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    act = model.act
    B, F, H, W = w.batch, w.frames, w.height, w.width
    ctx = to_device(inp["ctx"], act)
    lat = to_device(inp["noise"], act)
    img_ctx = None
    keep = None
    if w.i2v:
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
    ws = torch.empty(wan.workspace_bytes(cfg, B, w.tokens, w.text_len, w.img_len), dtype=torch.uint8, device="cuda")
    return cfg, model, lat, ctx, img_ctx, keep, ws


def _token_values(v, rows, w):
    """v [16, F, H, W] -> the head outputs [len(rows), 64] of the given tokens."""
    Hh, Wh = w.height // 2, w.width // 2
    f, i, j = rows // (Hh * Wh), (rows // Wh) % Hh, rows % Wh
    out = np.empty((len(rows), w.out_ch * 4))
    for c in range(w.out_ch):
        for ph in range(2):
            for pw in range(2):
                out[:, c * 4 + ph * 2 + pw] = v[c, f, 2 * i + ph, 2 * j + pw]
    return out


@pytest.mark.parametrize("name", ["wan13b_480p_block", "wan13b_480p_i2v_block", "wan14b_720p_block"])
def test_full_size_step_sampled_rows(wan, name):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0, block_input=False, zero_wx=False)
    cfg, model, lat, ctx, img_ctx, keep, ws = _setup(wan, w, inp)
    t = torch.from_numpy(inp["t"]).cuda()
    v = torch.empty(w.batch, w.out_ch, w.frames, w.height, w.width, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(cfg, lat, t, model.stack_table, model.block_tables, ctx, img_ctx, v, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    vh = v.cpu().numpy()
    img_np = None
    if w.i2v:
        img_np = O.image_context_mlp(inp["img_feat"][0], *(inp[k] for k in ["w_i1", "b_i1", "w_i2", "b_i2",
                                                                             "w_i3", "b_i3"]))
        assert rel_err(img_ctx[0].float().cpu().numpy(), img_np) <= BF16_TOL
    del model, ws
    torch.cuda.empty_cache()
    rows = sample_rows(w.tokens)
    lat_np = inp["noise"][0]
    if w.i2v:
        lat_np = O.i2v_input(inp["noise"][0], inp["cond"][0], O.i2v_mask(keep[0], w.frames, w.height, w.width))
    x = O.patchify(lat_np, inp["w_p"], inp["b_p"])
    e = O.time_mlp(float(inp["t"][0]), inp["w_t1"], inp["b_t1"], inp["w_t2"], inp["b_t2"])
    xr, parts = O.dit_block(x, e, inp["blocks"][0], inp["ctx"][0], w.heads, img_ctx=img_np, rows=rows,
                            return_parts=True)
    ref = O.head(xr, inp["w_head"], inp["b_head"])
    got = _token_values(vh[0], rows, w)
    err = rel_err(got, ref)
    print(f"{name}: head-output rel err {err:.3e} on {len(rows)} rows")
    assert err <= BF16_TOL


@pytest.mark.parametrize("name", ["wan13b_480p_block", "wan14b_720p_block"])
def test_full_size_block_call_sampled_rows(wan, name):
    """wan_dit_block_fwd alone on the residual-stream input: block output and the branch
    delta on the sampled rows."""
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=1, block_input=True)
    cfg, model, lat, ctx, img_ctx, keep, ws = _setup(wan, w, inp)
    from video_diffusion_transformer_wan_b200.model import to_device
    x = to_device(inp["x"], torch.float32)
    e = to_device(inp["e"], torch.float32)
    wan.dit_block_fwd(cfg, x, e, ctx, None, model.block_tables[0], ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    rows = sample_rows(w.tokens)
    got = x[0, torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    del model, ws, x
    torch.cuda.empty_cache()
    ref = O.dit_block(inp["x"][0], inp["e"][0], inp["blocks"][0], inp["ctx"][0], w.heads, rows=rows)
    x0 = inp["x"][0][rows]
    assert rel_err(got, ref) <= BF16_TOL
    derr = rel_err(got - x0, ref - x0)
    print(f"{name}: block delta rel err {derr:.3e}")
    assert derr <= BF16_TOL


def stack30_small():
    return dataclasses.replace(WORKLOADS["wan13b_480p_stack30"], frames=3, height=12, width=16)


def test_stack30_reduced_tokens_matches_oracle(wan):
    """The 30-block 1.3B stack (full width, 30 distinct per-block biases, one shared
    timestep MLP) with one rectified-flow velocity evaluation, at 144 tokens."""
    w = stack30_small()
    inp = make_inputs(w, seed=0, block_input=False)
    cfg, model, lat, ctx, img_ctx, keep, ws = _setup(wan, w, inp)
    from video_diffusion_transformer_wan_b200.model import to_device
    x1 = to_device(inp["x1"], model.act)
    x0 = lat
    u = torch.from_numpy(inp["u"]).cuda()
    xt = torch.empty_like(x1)
    t = torch.empty(w.batch, dtype=torch.float32, device="cuda")
    wan.flow_matching_input(cfg, x1, x0, u, xt, t)
    v = torch.empty(w.batch, 16, w.frames, w.height, w.width, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(cfg, xt, t, model.stack_table, model.block_tables, ctx, None, v, ws)
    loss = torch.empty(w.batch, dtype=torch.float32, device="cuda")
    wan.flow_matching_loss(cfg, v, x1, x0, loss)
    torch.cuda.synchronize()
    xt_ref = O.flow_matching_input(inp["x1"][0], inp["noise"][0], float(inp["u"][0]))
    ref = O.dit_stack(xt_ref, 1000.0 * float(inp["u"][0]), inp, inp["blocks"], inp["ctx"][0], w.heads)
    err = rel_err(v[0].cpu().numpy(), ref)
    print(f"stack30 at {w.tokens} tokens: rel err {err:.3e}")
    assert err <= BF16_TOL
    ref_loss = np.mean((ref - O.flow_matching_target(inp["x1"][0], inp["noise"][0])) ** 2)
    assert abs(float(loss[0]) - ref_loss) / ref_loss < 2e-2


GOLDEN_STACK30 = os.path.join(os.path.dirname(__file__), "golden", "wan13b_480p_stack30_seed0_velocity_rows.npz")


@pytest.fixture(scope="module")
def stack30_inputs():
    return make_inputs(WORKLOADS["wan13b_480p_stack30"], seed=0, block_input=False)


def test_stack30_full_size_matches_stored_oracle_velocity(wan, stack30_inputs):
    """The 30-block 1.3B stack at 480P, 81 frames (32760 tokens) with one rectified-flow
    velocity evaluation, through flow_matching_input and wan_dit_stack_fwd, against the
    oracle's velocity of the 256 sampled tokens (rows 0 and L-1 and the ragged last tile
    included), written by tests/golden/make_stack30_velocity.py (float32 products,
    float64 reductions: ~1e-6 from the float64 definition)."""
    g = np.load(GOLDEN_STACK30)
    w = WORKLOADS["wan13b_480p_stack30"]
    inp = stack30_inputs
    assert str(g["digest"]) == input_digest(inp), "input recipe changed: regenerate the stored velocity"
    rows = sample_rows(w.tokens)
    assert np.array_equal(g["rows"], rows)
    cfg, model, lat, ctx, img_ctx, keep, ws = _setup(wan, w, inp)
    from video_diffusion_transformer_wan_b200.model import to_device
    x1 = to_device(inp["x1"], model.act)
    u = torch.from_numpy(inp["u"]).cuda()
    xt = torch.empty_like(x1)
    t = torch.empty(w.batch, dtype=torch.float32, device="cuda")
    wan.flow_matching_input(cfg, x1, lat, u, xt, t)
    v = torch.empty(w.batch, 16, w.frames, w.height, w.width, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(cfg, xt, t, model.stack_table, model.block_tables, ctx, None, v, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = _token_values(v[0].cpu().numpy(), rows, w)
    del model, ws
    torch.cuda.empty_cache()
    err, rms = rel_err(got, g["values"]), rms_err(got, g["values"])
    print(f"stack30 at {w.tokens} tokens, 30 blocks: max rel err {err:.3e}, rms {rms:.3e}")
    assert err <= BF16_TOL


def test_stack30_full_size_properties(wan, stack30_inputs):
    """Full-size 30-block stack: (1) with every block's weights zero, each block is the
    identity and the output is head(LN(patchify)) - row-local, so the oracle checks it
    on sampled tokens; (2) the stack with real weights equals 30 consecutive block calls
    between a patchify/timestep-MLP call and the head call, bitwise."""
    w = WORKLOADS["wan13b_480p_stack30"]
    inp = stack30_inputs
    cfg, model, lat, ctx, img_ctx, keep, ws = _setup(wan, w, inp)
    B, F, H, W, L, D = w.batch, w.frames, w.height, w.width, w.tokens, w.dim
    t = torch.from_numpy((1000.0 * inp["u"]).astype(np.float32)).cuda()
    # (2) stack == parts
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    wan.dit_stack_fwd(cfg, lat, t, model.stack_table, model.block_tables, ctx, None, v, ws)
    x = torch.empty(B, L, D, dtype=torch.float32, device="cuda")
    e = torch.empty(B, 6, D, dtype=torch.float32, device="cuda")
    s = model.stack
    wan.patchify(cfg, lat, s["w_p"], s["b_p"], x, ws)
    wan.time_mlp(cfg, t, model.time_table, e)
    for bw in model.block_tables:
        wan.dit_block_fwd(cfg, x, e, ctx, None, bw, ws)
    v2 = torch.empty_like(v)
    wan.head_fwd(cfg, x, F, H, W, s["w_head"], s["b_head"], v2, ws)
    torch.cuda.synchronize()
    assert torch.equal(v, v2)
    assert torch.isfinite(v).all()
    # (1) zero blocks
    zero = {k: torch.zeros_like(val) for k, val in model.blocks[0].items()}
    zt = wan.block_weights(zero)
    wan.dit_stack_fwd(cfg, lat, t, model.stack_table, [zt] * w.n_blocks, ctx, None, v, ws)
    torch.cuda.synchronize()
    vh = v[0].cpu().numpy()
    rows = sample_rows(L)
    xr = O.patchify(inp["noise"][0], inp["w_p"], inp["b_p"])[rows]
    ref = O.head(xr, inp["w_head"], inp["b_head"])
    got = _token_values(vh, rows, w)
    assert rel_err(got, ref) <= BF16_TOL
