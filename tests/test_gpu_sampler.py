"""Parity of the generation loop (rectified-flow Euler steps with classifier-free
guidance, the DiT as the velocity model) with the CPU oracle, T2V and I2V, at sizes
the oracle finishes in seconds; plus the special cases that reduce the loop to one
stack call through the ABI."""
import numpy as np
import pytest

from oracle import wan_oracle as O
from gpu_util import BF16_TOL, host, rel_err
from test_gpu_block import Run, small_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wan():
    import video_diffusion_transformer_wan_b200 as w
    return w


def _input(wan, r, i2v):
    """The sampler input [B, in_ch, F, H, W]: noise, and for I2V the condition latent and
    the frame mask (first frame kept) built on the GPU; plus the oracle's fixed
    condition channels per sample."""
    w = r.w
    B, F, H, W = w.batch, w.frames, w.height, w.width
    noise = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    if not i2v:
        return noise, [None] * B
    keep = np.zeros((B, 1 + 4 * (F - 1)), np.uint8)
    keep[:, 0] = 1
    cond = torch.from_numpy(r.inp["cond"]).cuda().to(r.act)
    inp = torch.empty(B, 36, F, H, W, dtype=r.act, device="cuda")
    wan.i2v_input(r.cfg, noise, cond, torch.from_numpy(keep).cuda(), inp)
    cc = [O.i2v_input(r.inp["noise"][b], r.inp["cond"][b], O.i2v_mask(keep[b], F, H, W))[16:] for b in range(B)]
    return inp, cc


def _sample(wan, r, inp, n_steps, g, ctx=None, ctx_uncond=None, cache=None):
    B, _, F, H, W = inp.shape
    ctx = r.ctx if ctx is None else ctx
    ctx_uncond = r.ctx_uncond if ctx_uncond is None else ctx_uncond
    Li = 0 if r.img_ctx is None else r.img_ctx.shape[1]
    ws = torch.empty(wan.sample_workspace_bytes(r.cfg, len(r.model.block_tables), B, F, H, W, r.w.text_len, Li,
                                                cache), dtype=torch.uint8, device="cuda")
    out = torch.full((B, 16, F, H, W), float("nan"), dtype=torch.float32, device="cuda")
    wan.sample_euler_cfg(r.cfg, inp, n_steps, g, r.model.stack_table, r.model.block_tables, ctx, ctx_uncond,
                         r.img_ctx, out, ws, cache=cache)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    return out


@pytest.mark.parametrize("i2v", [False, True])
def test_sampler_matches_oracle(wan, i2v):
    """Four guided Euler steps (guidance 5) over two samples and two blocks; the final
    latent and the displacement x(1) - x(0) against the fp64 loop."""
    w = small_bf16(i2v=i2v, n_blocks=2, batch=2)
    r = Run(wan, w, zero_wx=False, uncond=True)
    inp, cc = _input(wan, r, i2v)
    n_steps, g = 4, 5.0
    got = host(_sample(wan, r, inp, n_steps, g))
    for b in range(w.batch):
        x0 = r.inp["noise"][b]
        ref = O.sample_euler_cfg(x0, n_steps, g, r.inp, r.inp["blocks"], r.inp["ctx"][b], r.inp["ctx_uncond"][b],
                                 w.heads, img_ctx=None if r.img_np is None else r.img_np[b], cond_channels=cc[b])
        e_x, e_d = rel_err(got[b], ref), rel_err(got[b] - x0, ref - x0)
        print(f"sampler i2v={i2v} b={b}: latent {e_x:.2e} displacement {e_d:.2e}")
        assert e_x <= BF16_TOL
        # The displacement sum_k dt (v_u + g (v_c - v_u)) is held to the same bf16 bar
        # (guidance amplifies the branch difference, not the rounding of the stack).
        assert e_d <= BF16_TOL


@pytest.mark.parametrize("g", [1.0, 0.0])
def test_one_step_is_one_stack_call(wan, g):
    """One step from t = 0: guidance 1 gives x0 + v_cond(x0, 0), guidance 0 gives
    x0 + v_uncond(x0, 0), with v from the stack call through the ABI on the same
    batch (the sampler's 2B-sample pass computes each sample's rows the same way)."""
    w = small_bf16(n_blocks=2, batch=2)
    r = Run(wan, w, zero_wx=False, uncond=True)
    inp, _ = _input(wan, r, False)
    got = _sample(wan, r, inp, 1, g)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    t = torch.zeros(B, dtype=torch.float32, device="cuda")
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    ctx = r.ctx if g == 1.0 else r.ctx_uncond
    wan.dit_stack_fwd(r.cfg, inp, t, r.model.stack_table, r.model.block_tables, ctx, None, v, r.ws)
    torch.cuda.synchronize()
    want = inp.float() + v
    assert (got - want).abs().max().item() <= 1e-6 * want.abs().max().item()


def test_sampler_deterministic_and_batch_independent(wan):
    """Same inputs give bitwise the same latent; a sample's result does not depend on
    the other samples of the batch."""
    w = small_bf16(n_blocks=1, batch=2)
    r = Run(wan, w, zero_wx=False, uncond=True)
    inp, _ = _input(wan, r, False)
    a = _sample(wan, r, inp, 3, 4.0)
    b = _sample(wan, r, inp, 3, 4.0)
    assert torch.equal(a, b)
    one = _sample(wan, r, inp[1:].contiguous(), 3, 4.0, r.ctx[1:].contiguous(), r.ctx_uncond[1:].contiguous())
    assert torch.equal(one[0], a[1])


@pytest.mark.parametrize("i2v", [False, True])
def test_cached_sampler_matches_oracle(wan, i2v):
    """Six steps with the diffusion cache (attention reused on steps 2, 4; unconditional
    pass skipped on steps 4, 5): against the oracle's cached loop, same schedule."""
    w = small_bf16(i2v=i2v, n_blocks=2, batch=2)
    r = Run(wan, w, zero_wx=False, uncond=True)
    inp, cc = _input(wan, r, i2v)
    n_steps, g = 6, 5.0
    pol = (1, 2, 3, 3)    # attn_start, attn_interval, cfg_start, cfg_interval
    sched = O.diffusion_cache_schedule(n_steps, *pol)
    assert [k for k, (a, _) in enumerate(sched) if a] == [2, 4] and [k for k, (_, c) in enumerate(sched) if c] == [4, 5]
    got = host(_sample(wan, r, inp, n_steps, g, cache=wan.DiffusionCache(*pol)))
    for b in range(w.batch):
        x0 = r.inp["noise"][b]
        ref = O.sample_euler_cfg_cached(x0, n_steps, g, r.inp, r.inp["blocks"], r.inp["ctx"][b],
                                        r.inp["ctx_uncond"][b], w.heads, sched,
                                        img_ctx=None if r.img_np is None else r.img_np[b], cond_channels=cc[b])
        e_x, e_d = rel_err(got[b], ref), rel_err(got[b] - x0, ref - x0)
        print(f"cached sampler i2v={i2v} b={b}: latent {e_x:.2e} displacement {e_d:.2e}")
        assert e_x <= BF16_TOL
        assert e_d <= BF16_TOL


def test_cache_without_reuse_is_the_plain_loop(wan):
    """Intervals of 1 never reuse: bitwise the loop without a cache."""
    w = small_bf16(n_blocks=2, batch=2)
    r = Run(wan, w, zero_wx=False, uncond=True)
    inp, _ = _input(wan, r, False)
    a = _sample(wan, r, inp, 3, 4.0)
    b = _sample(wan, r, inp, 3, 4.0, cache=wan.DiffusionCache(0, 1, 0, 1))
    assert torch.equal(a, b)
