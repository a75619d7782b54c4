"""FP8 (E4M3) path through the C ABI against the oracle: quantisation codes and scales
bit-exact (same float32 input, same float32 decision), the kind::f8f6f4 GEMM against
the product of the codes, the FP8 block against the oracle's FP8 block (T2V, I2V,
and the 1.3B 480P block on sampled rows), and 8-bit attention (operand codes bit-exact,
output against the oracle's running-base option within the derived bars)."""
import numpy as np
import pytest

from oracle import wan_oracle as O
from wan_inputs import WORKLOADS, make_inputs, round_bf16, sample_rows
from gpu_util import (FP8_ATTN_RB_TOL_MAX, FP8_ATTN_RB_TOL_RMS, attention_split_units, sample_warps,
                      FP8A_BLOCK_TOL_MAX, FP8A_BLOCK_TOL_RMS, FP8_SAMPLE_TOL_MAX, FP8_SAMPLE_TOL_RMS, FP8_STACK_TOL_MAX,
                      FP8_STACK_TOL_RMS, FP8_TOL_MAX, FP8_TOL_RMS, dev, host, rel_err, rms_err, rng)
from test_gpu_block import Run, small_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

E4M3 = np.array([O.e4m3_decode(c) for c in range(256)])


@pytest.fixture(scope="module")
def wan():
    import video_diffusion_transformer_wan_b200 as w
    return w


def _cfg(wan, dtype="bf16"):
    return wan.make_config(128, 1, 128, dtype=dtype)


def _rows_input(seed, M, K):
    r = rng(seed)
    a = r.standard_normal((M, K)) * np.exp2(r.integers(-12, 10, (M, 1)))
    a[1] = 0.0                                   # all-zero row: scale 1
    a[2, :7] = [448.0, -1e-8, 3e-5, 2 ** -9, 1.5 * 2 ** -9, 17.0, -19.0]
    return a


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K", [(37, 1536), (5, 8960), (300, 64)])
def test_quantize_rows_bit_exact(wan, dtype, M, K):
    a = _rows_input(M + K, M, K)
    a = round_bf16(a) if dtype == "bf16" else a.astype(np.float32)
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    wan.fp8_quantize_rows(_cfg(wan, dtype), dev(a, act), q, s)
    torch.cuda.synchronize()
    ref_q, ref_s = O.quantize_e4m3(np.asarray(a, np.float32), axis=-1)
    assert np.array_equal(s.cpu().numpy(), ref_s[:, 0])
    assert np.array_equal(E4M3[q.cpu().numpy()], ref_q)


def test_quantize_tensor_bit_exact(wan):
    w = round_bf16(0.02 * rng(3).standard_normal((384, 1536)))
    q = torch.empty(w.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    wan.fp8_quantize_tensor(_cfg(wan), dev(w, torch.bfloat16), q, s)
    torch.cuda.synchronize()
    ref_q, ref_s = O.quantize_e4m3(np.asarray(w, np.float32))
    assert s.item() == float(ref_s)
    assert np.array_equal(E4M3[q.cpu().numpy()], ref_q)


@pytest.mark.parametrize("M,N,K,epi", [(333, 1536, 1536, "store"), (300, 256, 8960, "f32"), (129, 64, 512, "f32"),
                                       (200, 128, 1536, "store"), (257, 1536, 1536, "residual"),
                                       (130, 4608, 1536, "gelu")])
def test_linear_fp8(wan, M, N, K, epi):
    r = rng(M * 7 + N + K)
    x = round_bf16(r.standard_normal((M, K)))
    w = round_bf16(0.02 * r.standard_normal((N, K)))
    b = round_bf16(0.1 * r.standard_normal(N))
    cfg = _cfg(wan)
    xq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    xs = torch.empty(M, dtype=torch.float32, device="cuda")
    wq = torch.empty(N, K, dtype=torch.uint8, device="cuda")
    ws = torch.empty(1, dtype=torch.float32, device="cuda")
    wan.fp8_quantize_rows(cfg, dev(x, torch.bfloat16), xq, xs)
    wan.fp8_quantize_tensor(cfg, dev(w, torch.bfloat16), wq, ws)
    ref = O.linear_fp8(x, w, b)
    kind = {"store": wan.EPI_STORE, "gelu": wan.EPI_GELU, "f32": wan.EPI_F32, "residual": wan.EPI_RESIDUAL}[epi]
    gate = gate_b = None
    if epi in ("store", "gelu"):
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    elif epi == "f32":
        out = torch.empty(M, N, dtype=torch.float32, device="cuda")
    else:
        x0 = r.standard_normal((M, N)).astype(np.float32)
        g = r.standard_normal(N).astype(np.float32)
        out = torch.from_numpy(x0).cuda()
        gate = torch.from_numpy(g).cuda()
        ref = x0 + g * ref
    wan.linear_fp8_fwd(cfg, xq, xs, wq, ws, dev(b, torch.bfloat16), out, kind, gate=gate,
                       rows_per_batch=M)
    torch.cuda.synchronize()
    if epi == "gelu":
        ref = O.gelu_tanh(ref)
    tol = 1e-4 if epi in ("f32", "residual") else 8e-3          # fp32 accumulation; bf16 output rounding
    assert rel_err(host(out), ref) <= tol


@pytest.mark.parametrize("i2v", [False, True])
def test_block_fp8_matches_oracle(wan, i2v):
    from video_diffusion_transformer_wan_b200.model import Fp8Block
    w = small_bf16(i2v=i2v, dim=512, heads=4, ffn=1024)
    r = Run(wan, w, zero_wx=False)
    fb = Fp8Block(r.cfg, r.model.blocks[0])
    ws = torch.empty(wan.fp8_workspace_bytes(r.cfg, w.batch, w.tokens, w.text_len, w.img_len if i2v else 0),
                     dtype=torch.uint8, device="cuda")
    x = r.x.clone()
    wan.dit_block_fp8_fwd(r.cfg, x, r.e, r.ctx, r.img_ctx, fb.table, fb.scale_table, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(x)
    for b in range(w.batch):
        img = None if r.img_np is None else r.img_np[b]
        ref = O.dit_block(r.inp["x"][b], r.inp["e"][b], r.inp["blocks"][0], r.inp["ctx"][b], w.heads, img_ctx=img,
                          fp8=True)
        d_got, d_ref = got[b] - r.inp["x"][b], ref - r.inp["x"][b]
        print(f"fp8 block i2v={i2v} b={b}: max {rel_err(d_got, d_ref):.2e} rms {rms_err(d_got, d_ref):.2e}")
        assert rel_err(d_got, d_ref) <= FP8_TOL_MAX
        assert rms_err(d_got, d_ref) <= FP8_TOL_RMS


def test_block_fp8_full_size_sampled_rows(wan):
    """The 1.3B 480P block (L = 32760) in FP8, 256 sampled rows against the oracle."""
    from video_diffusion_transformer_wan_b200.model import DitModel, Fp8Block, config_for, to_device
    w = WORKLOADS["wan13b_480p_block"]
    inp = make_inputs(w, seed=0)
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    fb = Fp8Block(cfg, model.blocks[0])
    x = to_device(inp["x"], torch.float32)
    e = to_device(inp["e"], torch.float32)
    ctx = to_device(inp["ctx"], torch.bfloat16)
    ws = torch.empty(wan.fp8_workspace_bytes(cfg, 1, w.tokens, w.text_len), dtype=torch.uint8, device="cuda")
    wan.dit_block_fp8_fwd(cfg, x, e, ctx, None, fb.table, fb.scale_table, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    rows = sample_rows(w.tokens)
    got = x[0].cpu().numpy().astype(np.float64)[rows]
    ref = O.dit_block(inp["x"][0], inp["e"][0], inp["blocks"][0], inp["ctx"][0], w.heads, rows=rows, fp8=True)
    d_got, d_ref = got - inp["x"][0][rows], ref - inp["x"][0][rows]
    print(f"fp8 block 1.3B sampled rows: max {rel_err(d_got, d_ref):.2e} rms {rms_err(d_got, d_ref):.2e}")
    assert rel_err(d_got, d_ref) <= FP8_TOL_MAX
    assert rms_err(d_got, d_ref) <= FP8_TOL_RMS


def _fp8_run(wan, i2v=False, batch=2, n_blocks=2, attention_fp8=False):
    from video_diffusion_transformer_wan_b200.model import Fp8Block
    w = small_bf16(i2v=i2v, dim=512, heads=4, ffn=1024, n_blocks=n_blocks, batch=batch)
    r = Run(wan, w, zero_wx=False, uncond=True)
    fbs = [Fp8Block(r.cfg, b, attention_fp8=attention_fp8) for b in r.model.blocks]
    return w, r, fbs


# The stack and sampler bars hold with 8-bit self-attention as well: the derivation of
# FP8_STACK_TOL_* / FP8_SAMPLE_TOL_* with q, k and v also moved by +-2^-9 and the
# running base emulated gives <= 0.79 % / 0.54 % (stack, 8 trials per sample) and
# <= 1.22 % / 1.0 % (3-step sampler displacement, 4 trials).
@pytest.mark.parametrize("i2v,fa", [(False, False), (True, False), (False, True)])
def test_stack_fp8_matches_oracle(wan, i2v, fa):
    """Patchify, time MLP, two FP8 blocks (with 8-bit self-attention if fa), head: the
    velocity against the oracle's FP8 stack."""
    w, r, fbs = _fp8_run(wan, i2v, attention_fp8=fa)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    t = torch.from_numpy(r.inp["t"]).cuda()
    lat = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    if i2v:
        lat = torch.cat([lat, torch.zeros(B, 20, F, H, W, dtype=r.act, device="cuda")], dim=1).contiguous()
    v = torch.empty(B, 16, F, H, W, dtype=torch.float32, device="cuda")
    ws = torch.empty(wan.fp8_workspace_bytes(r.cfg, B, w.tokens, w.text_len, w.img_len if i2v else 0),
                     dtype=torch.uint8, device="cuda")
    wan.dit_stack_fp8_fwd(r.cfg, lat, t, r.model.stack_table, [f.table for f in fbs], [f.scale_table for f in fbs],
                          r.ctx, r.img_ctx, v, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(v)
    for b in range(B):
        lat_np = r.inp["noise"][b]
        if i2v:
            lat_np = np.concatenate([lat_np, np.zeros((20, F, H, W))], axis=0)
        ref = O.dit_stack(lat_np, float(r.inp["t"][b]), r.inp, r.inp["blocks"], r.inp["ctx"][b], w.heads,
                          img_ctx=None if r.img_np is None else r.img_np[b], fp8=True, fp8_attention=fa)
        print(f"fp8 stack i2v={i2v} attn8={fa} b={b}: max {rel_err(got[b], ref):.2e} rms {rms_err(got[b], ref):.2e}")
        assert rel_err(got[b], ref) <= FP8_STACK_TOL_MAX
        assert rms_err(got[b], ref) <= FP8_STACK_TOL_RMS


@pytest.mark.parametrize("fa", [False, True])
def test_sampler_fp8_matches_oracle(wan, fa):
    """Three guided Euler steps with FP8 linear layers (including the cached context
    K|V projections; with 8-bit self-attention if fa) against the oracle's FP8 loop."""
    w, r, fbs = _fp8_run(wan, attention_fp8=fa)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    inp = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    ws = torch.empty(wan.sample_workspace_bytes(r.cfg, 2, B, F, H, W, w.text_len, 0, None, fp8=True),
                     dtype=torch.uint8, device="cuda")
    out = torch.full((B, 16, F, H, W), float("nan"), dtype=torch.float32, device="cuda")
    wan.sample_euler_cfg(r.cfg, inp, 3, 5.0, r.model.stack_table, [f.table for f in fbs], r.ctx, r.ctx_uncond, None,
                         out, ws, fp8_scales=[f.scale_table for f in fbs])
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(out)
    for b in range(B):
        x0 = r.inp["noise"][b]
        ref = O.sample_euler_cfg(x0, 3, 5.0, r.inp, r.inp["blocks"], r.inp["ctx"][b], r.inp["ctx_uncond"][b],
                                 w.heads, fp8=True, fp8_attention=fa)
        d_got, d_ref = got[b] - x0, ref - x0
        print(f"fp8 sampler attn8={fa} b={b}: displacement max {rel_err(d_got, d_ref):.2e} rms {rms_err(d_got, d_ref):.2e}")
        assert rel_err(d_got, d_ref) <= FP8_SAMPLE_TOL_MAX
        assert rms_err(d_got, d_ref) <= FP8_SAMPLE_TOL_RMS


# ----------------------------------------------------------------------------------------
# 8-bit attention
# ----------------------------------------------------------------------------------------

def _qkv(seed, B, Lq, Lk, H, logit_std):
    r = rng(seed)
    s = np.sqrt(logit_std)
    D = H * 128
    q = round_bf16(r.standard_normal((B, Lq, D)) * s * np.exp2(r.integers(-3, 4, (B, Lq, 1))))
    k = round_bf16(r.standard_normal((B, Lk, D)) * s)
    v = round_bf16(r.standard_normal((B, Lk, D)))
    return q, k, v


def _attn_cfg(wan, H):
    return wan.make_config(H * 128, H, 4 * H * 128)


@pytest.mark.parametrize("B,Lq,Lk,H", [(2, 300, 700, 2), (1, 1, 65, 1), (1, 129, 1, 3)])
def test_attention_fp8_quantize_bit_exact(wan, B, Lq, Lk, H):
    q, k, v = _qkv(B * Lq + Lk, B, Lq, Lk, H, 1.0)
    q[0, 0, :128] = 0.0                                  # a zero (row, head): scale 1
    D = H * 128
    S = (Lk + 63) // 64 * 64
    qc = torch.empty(B, Lq, D, dtype=torch.uint8, device="cuda")
    qs = torch.empty(B, Lq, H, dtype=torch.float32, device="cuda")
    kc = torch.empty(B, Lk, D, dtype=torch.uint8, device="cuda")
    vt = torch.full((B, D, S), 0xAB, dtype=torch.uint8, device="cuda")
    kvs = torch.empty(B, H, 2, dtype=torch.float32, device="cuda")
    bf = torch.bfloat16
    wan.attention_fp8_quantize(_attn_cfg(wan, H), dev(q, bf), dev(k, bf), dev(v, bf), H, 128, qc, qs, kc, vt, kvs)
    torch.cuda.synchronize()
    qc, qs, kc, vt, kvs = (t.cpu().numpy() for t in (qc, qs, kc, vt, kvs))
    for b in range(B):
        for h in range(H):
            sl = slice(h * 128, (h + 1) * 128)
            rq, rs = O.quantize_e4m3(np.asarray(q[b][:, sl], np.float32), axis=-1)
            assert np.array_equal(E4M3[qc[b][:, sl]], rq) and np.array_equal(qs[b][:, h], rs[:, 0])
            rk, sk = O.quantize_e4m3(np.asarray(k[b][:, sl], np.float32))
            assert np.array_equal(E4M3[kc[b][:, sl]], rk) and kvs[b, h, 0] == sk
            rv, sv = O.quantize_e4m3(np.asarray(v[b][:, sl], np.float32))
            assert np.array_equal(E4M3[vt[b][sl, :Lk]], rv.T) and kvs[b, h, 1] == sv
            assert not vt[b][sl, Lk:].any()              # keys past Lk are code 0 up to the 64-multiple


def _attention_fp8_case(wan, B, Lq, Lk, H, logit_std, seed, rows=None):
    """The kernel against the oracle's running-base option (the kernel's bases and its
    key-split units) at the bf16-level bar, and against the definition (the final row
    maximum as the base) at the bar derived for the subnormal range."""
    q, k, v = _qkv(seed, B, Lq, Lk, H, logit_std)
    D = H * 128
    cfg = _attn_cfg(wan, H)
    bf = torch.bfloat16
    o = torch.full((B, Lq, D), float("nan"), dtype=bf, device="cuda")
    ws = torch.empty(wan.attention_fp8_workspace_bytes(cfg, B, Lq, Lk), dtype=torch.uint8, device="cuda")
    wan.attention_fp8_fwd(cfg, dev(q, bf), dev(k, bf), dev(v, bf), o, H, 128, ws=ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(o)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    split = attention_split_units(B, H, Lq, Lk, nsm)
    r = np.arange(Lq) if rows is None else rows
    for b in range(B):
        ref_rb = O.attention_fp8(q[b], k[b], v[b], H, running_base=True, split_units=split[b], rows=r)
        e_max, e_rms = rel_err(got[b][r], ref_rb), rms_err(got[b][r], ref_rb)
        print(f"8-bit attention B={B} Lq={Lq} Lk={Lk} H={H} std={logit_std} split={len(split[b])}: "
              f"running-base oracle max {e_max:.2e} rms {e_rms:.2e}")
        assert e_max <= FP8_ATTN_RB_TOL_MAX
        assert e_rms <= FP8_ATTN_RB_TOL_RMS
        ref = O.attention_fp8(q[b][r], k[b], v[b], H)
        print(f"  against the definition's final-maximum base: max {rel_err(got[b][r], ref):.2e} "
              f"rms {rms_err(got[b][r], ref):.2e}")
    return got, q, k, v


@pytest.mark.parametrize("B,Lq,Lk,H,logit_std", [
    (1, 300, 700, 2, 1.0),        # two query-tile pairs, ragged; 6 key tiles, ragged
    (1, 300, 700, 2, 4.0),        # peaked rows: the running base moves
    (2, 257, 2100, 2, 1.0),       # 17 key tiles: the partial last wave is split over the keys
    (1, 130, 1, 1, 1.0),          # one key
    (1, 1, 300, 2, 0.36),         # one query
])
def test_attention_fp8_parity(wan, B, Lq, Lk, H, logit_std):
    _attention_fp8_case(wan, B, Lq, Lk, H, logit_std, seed=Lq * 7 + Lk)


@pytest.mark.parametrize("L,H", [(32760, 12), (75600, 40)])
def test_attention_fp8_full_size_sampled_rows(wan, L, H):
    """1.3B (32760 tokens, 12 heads) and 14B (75600 tokens, 40 heads) self-attention
    shapes on eight sampled 32-row groups (the first, the ragged last tile's, seeded
    ones): under the running base a row's result depends on its whole group."""
    rows = sample_warps(L)
    got, q, k, v = _attention_fp8_case(wan, 1, L, L, H, 1.0, seed=5, rows=rows)
    exact = O.attention(q[0][rows], k[0], v[0], H)
    assert rms_err(got[0][rows], exact) > 4 * FP8_ATTN_RB_TOL_RMS        # it is the 8-bit path, not bf16


@pytest.mark.parametrize("i2v", [False, True])
def test_block_fp8_attention_matches_oracle(wan, i2v):
    """FP8 block with 8-bit self-attention (960 tokens: 8 key tiles, so the running base
    moves) against the oracle's; the 8-bit attention path is the one that ran (its five
    quantiser launches)."""
    from video_diffusion_transformer_wan_b200.model import Fp8Block
    w = small_bf16(i2v=i2v, frames=5, height=24, width=32, dim=512, heads=4, ffn=1024)
    r = Run(wan, w, zero_wx=False)
    ws = torch.empty(wan.fp8_workspace_bytes(r.cfg, w.batch, w.tokens, w.text_len, w.img_len if i2v else 0),
                     dtype=torch.uint8, device="cuda")
    launches = {}
    outs = {}
    for fa in (False, True):
        fb = Fp8Block(r.cfg, r.model.blocks[0], attention_fp8=fa)
        x = r.x.clone()
        torch.cuda.synchronize()
        n0 = wan.launch_count()
        wan.dit_block_fp8_fwd(r.cfg, x, r.e, r.ctx, r.img_ctx, fb.table, fb.scale_table, ws)
        launches[fa] = wan.launch_count() - n0
        torch.cuda.synchronize()
        assert wan.device_status() == 0
        outs[fa] = host(x)
    assert launches[True] - launches[False] == 5
    for b in range(w.batch):
        img = None if r.img_np is None else r.img_np[b]
        ref = O.dit_block(r.inp["x"][b], r.inp["e"][b], r.inp["blocks"][0], r.inp["ctx"][b], w.heads, img_ctx=img,
                          fp8=True, fp8_attention=True)
        d_got, d_ref = outs[True][b] - r.inp["x"][b], ref - r.inp["x"][b]
        print(f"fp8 block + 8-bit attention i2v={i2v}: max {rel_err(d_got, d_ref):.2e} rms {rms_err(d_got, d_ref):.2e}")
        assert rel_err(d_got, d_ref) <= FP8A_BLOCK_TOL_MAX
        assert rms_err(d_got, d_ref) <= FP8A_BLOCK_TOL_RMS


def test_block_fp8_attention_full_size_sampled_rows(wan):
    """The 1.3B 480P block with FP8 linears and 8-bit self-attention, 256 sampled rows."""
    from video_diffusion_transformer_wan_b200.model import DitModel, Fp8Block, config_for, to_device
    w = WORKLOADS["wan13b_480p_block"]
    inp = make_inputs(w, seed=0)
    cfg = config_for(w)
    model = DitModel(cfg, inp)
    fb = Fp8Block(cfg, model.blocks[0], attention_fp8=True)
    x = to_device(inp["x"], torch.float32)
    e = to_device(inp["e"], torch.float32)
    ctx = to_device(inp["ctx"], torch.bfloat16)
    ws = torch.empty(wan.fp8_workspace_bytes(cfg, 1, w.tokens, w.text_len), dtype=torch.uint8, device="cuda")
    wan.dit_block_fp8_fwd(cfg, x, e, ctx, None, fb.table, fb.scale_table, ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    rows = sample_rows(w.tokens)
    got = x[0].cpu().numpy().astype(np.float64)[rows]
    ref = O.dit_block(inp["x"][0], inp["e"][0], inp["blocks"][0], inp["ctx"][0], w.heads, rows=rows, fp8=True,
                      fp8_attention=True)
    d_got, d_ref = got - inp["x"][0][rows], ref - inp["x"][0][rows]
    print(f"fp8 block + 8-bit attention 1.3B sampled rows: max {rel_err(d_got, d_ref):.2e} "
          f"rms {rms_err(d_got, d_ref):.2e}")
    assert rel_err(d_got, d_ref) <= FP8A_BLOCK_TOL_MAX
    assert rms_err(d_got, d_ref) <= FP8A_BLOCK_TOL_RMS


@pytest.mark.parametrize("fa", [False, True])
def test_cached_sampler_fp8_matches_oracle(wan, fa):
    """Six guided Euler steps with the diffusion cache (attention reused on steps 2, 4;
    unconditional pass skipped on steps 4, 5) and FP8 linear layers (and 8-bit
    self-attention if fa) against the oracle's cached FP8 loop. The FP8 sampler bars
    hold here too: the same derivation gives <= 1.34 % (max) and 0.95 % (RMS) on the
    displacement (4 trials each), 4.2 % RMS away from the bf16 cached loop."""
    w, r, fbs = _fp8_run(wan, attention_fp8=fa)
    B, F, H, W = w.batch, w.frames, w.height, w.width
    inp = torch.from_numpy(r.inp["noise"]).cuda().to(r.act)
    n_steps, g, pol = 6, 5.0, (1, 2, 3, 3)
    cache = wan.DiffusionCache(*pol)
    ws = torch.empty(wan.sample_workspace_bytes(r.cfg, 2, B, F, H, W, w.text_len, 0, cache, fp8=True),
                     dtype=torch.uint8, device="cuda")
    out = torch.full((B, 16, F, H, W), float("nan"), dtype=torch.float32, device="cuda")
    wan.sample_euler_cfg(r.cfg, inp, n_steps, g, r.model.stack_table, [f.table for f in fbs], r.ctx, r.ctx_uncond,
                         None, out, ws, cache=cache, fp8_scales=[f.scale_table for f in fbs])
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(out)
    sched = O.diffusion_cache_schedule(n_steps, *pol)
    for b in range(B):
        x0 = r.inp["noise"][b]
        ref = O.sample_euler_cfg_cached(x0, n_steps, g, r.inp, r.inp["blocks"], r.inp["ctx"][b],
                                        r.inp["ctx_uncond"][b], w.heads, sched, fp8=True, fp8_attention=fa)
        d_got, d_ref = got[b] - x0, ref - x0
        print(f"cached fp8 sampler attn8={fa} b={b}: max {rel_err(d_got, d_ref):.2e} rms {rms_err(d_got, d_ref):.2e}")
        assert rel_err(d_got, d_ref) <= FP8_SAMPLE_TOL_MAX
        assert rms_err(d_got, d_ref) <= FP8_SAMPLE_TOL_RMS


def test_attention_fp8_fused_qkv_layout(wan):
    """q, k and v as column slices of one [B, L, 3D] projection (row stride 3D, head
    columns from 0, D and 2D), and the output into a wider buffer at a column offset."""
    B, L, H = 2, 700, 2
    D = H * 128
    q, k, v = _qkv(11, B, L, L, H, 1.0)
    qkv = np.concatenate([q, k, v], axis=2)
    cfg = _attn_cfg(wan, H)
    bf = torch.bfloat16
    o = torch.full((B, L, D + 64), float("nan"), dtype=bf, device="cuda")
    ws = torch.empty(wan.attention_fp8_workspace_bytes(cfg, B, L, L), dtype=torch.uint8, device="cuda")
    t = dev(qkv, bf)
    wan.attention_fp8_fwd(cfg, t, t, t, o, H, 128, 0, D, 2 * D, 64, ws=ws)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    got = host(o)
    assert np.isnan(got[:, :, :64]).all()                                 # columns before o_col0 untouched
    split = attention_split_units(B, H, L, L, torch.cuda.get_device_properties(0).multi_processor_count)
    for b in range(B):
        ref = O.attention_fp8(q[b], k[b], v[b], H, running_base=True, split_units=split[b])
        assert rel_err(got[b][:, 64:], ref) <= FP8_ATTN_RB_TOL_MAX
        assert rms_err(got[b][:, 64:], ref) <= FP8_ATTN_RB_TOL_RMS
