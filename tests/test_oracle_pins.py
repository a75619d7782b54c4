"""Pins of the CPU oracle to facts outside itself (library routines, closed forms,
invariants, brute force, and the numbers the Wan 2.1 pages print).

Each pin is written as a ``check_*`` function that takes the oracle function(s)
under test, so ``test_oracle_mutations.py`` can plant plausible mistakes in the
oracle and show that some pin fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as tF

from oracle import wan_oracle as O
from wan_inputs import WORKLOADS, make_inputs, round_bf16, bf16_bits, bits_to_f32, sample_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = lambda s: np.random.Generator(np.random.PCG64(s))  # noqa: E731


def t64(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


# ----------------------------------------------------------------------------------------
# Golden: the pages' config table and shape formula
# ----------------------------------------------------------------------------------------

def test_token_count_matches_page_formula():
    g = json.load(open(os.path.join(GOLDEN, "wan21_config_table.json")))
    c = g["vae_compression"]
    for vid in g["videos"]:
        T = vid["T_plus_1"] - 1
        L_page = (1 + T // 4) * (vid["H"] // 16) * (vid["W"] // 16)   # pixel-space formula
        lat = (1 + T // c["t"], vid["H"] // c["h"], vid["W"] // c["w"])  # latent grid
        assert O.token_count(*lat) == L_page
    assert WORKLOADS["wan13b_480p_block"].tokens == 32760
    assert WORKLOADS["wan14b_720p_block"].tokens == 75600
    assert WORKLOADS["tiny_f32_block"].tokens == 32
    with pytest.raises(ValueError):
        O.token_count(2, 7, 8)


def _block_param_count(D, F):
    # self-attn qkv+o, cross-attn q+kv+o, FFN (weights and biases), per-block modulation bias
    return (3 * D * D + 3 * D) + (D * D + D) + (D * D + D) + (2 * D * D + 2 * D) + (D * D + D) \
        + (F * D + F) + (D * F + D) + 6 * D


def test_parameter_count_matches_model_names():
    """The block inventory (8 D^2 attention matrices, a plain 2-matrix FFN and a shared
    AdaLN MLP) reproduces the 1.3B / 14B names of the config table; a GLU FFN or an
    unshared AdaLN would not."""
    g = json.load(open(os.path.join(GOLDEN, "wan21_config_table.json")))
    for name, m in g["models"].items():
        D, F, n = m["dim"], m["ffn"], m["layers"]
        total = n * _block_param_count(D, F)
        assert abs(total / m["nominal_params"] - 1) < 0.08, (name, total)
        glu = n * (_block_param_count(D, F) + F * D)
        assert glu / m["nominal_params"] > 1.18
        unshared = n * 6 * D * D
        frac = unshared / (total + unshared)
        assert abs(frac - g["adaln_sharing_saves_fraction"]) < 0.07


# ----------------------------------------------------------------------------------------
# Patchify / unpatchify
# ----------------------------------------------------------------------------------------

def check_patchify(patchify):
    rng = RNG(1)
    for C, F, H, W, D in [(16, 2, 8, 8, 24), (36, 3, 6, 10, 7), (4, 1, 2, 2, 3)]:
        lat = rng.standard_normal((C, F, H, W))
        w = rng.standard_normal((D, C, 1, 2, 2))
        b = rng.standard_normal(D)
        ref = tF.conv3d(t64(lat)[None], t64(w), t64(b), stride=(1, 2, 2))[0]  # [D,F,H/2,W/2]
        ref = ref.permute(1, 2, 3, 0).reshape(-1, D).numpy()
        got = patchify(lat, w, b)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_patchify_is_the_strided_conv3d():
    check_patchify(O.patchify)


def check_patch_roundtrip(patchify, unpatchify):
    rng = RNG(2)
    C, F, H, W = 16, 3, 6, 10
    lat = rng.standard_normal((C, F, H, W))
    onehot = np.zeros((C * 4, C, 1, 2, 2))
    for c in range(C):
        for ph in range(2):
            for pw in range(2):
                onehot[c * 4 + ph * 2 + pw, c, 0, ph, pw] = 1.0
    tokens = patchify(lat, onehot, np.zeros(C * 4))
    # brute-force gather of one token
    f, i, j = 2, 1, 3
    tok = tokens[(f * (H // 2) + i) * (W // 2) + j]
    for c in range(C):
        assert tok[c * 4 + 0] == lat[c, f, 2 * i, 2 * j]
        assert tok[c * 4 + 3] == lat[c, f, 2 * i + 1, 2 * j + 1]
    back = unpatchify(tokens, C, F, H, W)
    assert np.array_equal(back, lat)           # exact permutation
    y = rng.standard_normal((F * (H // 2) * (W // 2), C * 4))
    assert np.array_equal(patchify(unpatchify(y, C, F, H, W), onehot, np.zeros(C * 4)), y)


def test_patchify_unpatchify_roundtrip_exact():
    check_patch_roundtrip(O.patchify, O.unpatchify)


# ----------------------------------------------------------------------------------------
# Timestep embedding, shared MLP, per-block bias
# ----------------------------------------------------------------------------------------

def check_sinusoid(emb_fn):
    e0 = emb_fn(0.0, 256)
    assert np.array_equal(e0, np.concatenate([np.ones(128), np.zeros(128)]))
    e = emb_fn(math.pi / 2, 256)                 # first frequency is 1: cos(pi/2)=0, sin(pi/2)=1
    assert abs(e[0]) < 1e-15 and abs(e[128] - 1) < 1e-15
    for t in [0.3, 17.0, 999.9]:
        e = emb_fn(t, 256)
        np.testing.assert_allclose(e[:128] ** 2 + e[128:] ** 2, 1.0, atol=1e-14)
        # independent route to the frequencies: exp(-ln(10000) i / 128)
        f = torch.exp(-math.log(10000.0) * torch.arange(128, dtype=torch.float64) / 128)
        ref = torch.cat([torch.cos(t * f), torch.sin(t * f)]).numpy()
        np.testing.assert_allclose(e, ref, atol=1e-12)


def test_sinusoid_closed_forms():
    check_sinusoid(O.sinusoidal_embedding)


def check_time_mlp(time_mlp, block_modulation):
    rng = RNG(3)
    D = 32
    w1, b1 = rng.standard_normal((D, 256)) * 0.1, rng.standard_normal(D) * 0.1
    w2, b2 = rng.standard_normal((6 * D, D)) * 0.1, rng.standard_normal(6 * D) * 0.1
    t = 431.5
    mlp = torch.nn.Sequential(torch.nn.Linear(256, D), torch.nn.SiLU(), torch.nn.Linear(D, 6 * D)).double()
    with torch.no_grad():
        mlp[0].weight.copy_(t64(w1)); mlp[0].bias.copy_(t64(b1))
        mlp[2].weight.copy_(t64(w2)); mlp[2].bias.copy_(t64(b2))
        ref = mlp(t64(O.sinusoidal_embedding(t, 256))).numpy().reshape(6, D)
    e = time_mlp(t, w1, b1, w2, b2)
    np.testing.assert_allclose(e, ref, rtol=1e-12, atol=1e-13)
    bias = rng.standard_normal((6, D))
    assert np.array_equal(block_modulation(e, bias), block_modulation(e, bias.copy()))  # equal biases
    delta = rng.standard_normal((6, D))
    np.testing.assert_allclose(block_modulation(e, bias + delta) - block_modulation(e, bias), delta,
                               atol=1e-13)


def test_shared_time_mlp_and_block_bias():
    check_time_mlp(O.time_mlp, O.block_modulation)


# ----------------------------------------------------------------------------------------
# LayerNorm, modulation, GELU, softmax
# ----------------------------------------------------------------------------------------

def check_layer_norm(ln):
    rng = RNG(4)
    x = rng.standard_normal((7, 96)) * 3 + 1.5
    ref = tF.layer_norm(t64(x), (96,), eps=1e-6).numpy()
    np.testing.assert_allclose(ln(x, 1e-6), ref, rtol=1e-12, atol=1e-12)
    y = ln(x, 1e-6)
    var = x.var(axis=-1)
    np.testing.assert_allclose(y.mean(axis=-1), 0.0, atol=1e-13)
    np.testing.assert_allclose((y ** 2).mean(axis=-1), var / (var + 1e-6), rtol=1e-12)
    c = np.full((2, 16), 3.25)                   # constant rows normalise to exactly 0
    assert np.array_equal(ln(c, 1e-6), np.zeros_like(c))


def test_layer_norm_pins():
    check_layer_norm(O.layer_norm)


def check_modulate(modulate, ln):
    rng = RNG(5)
    x = rng.standard_normal((5, 64))
    h = ln(x, 1e-6)
    z = np.zeros(64)
    np.testing.assert_array_equal(modulate(h, z, z), h)            # scale = shift = 0: plain LN
    sh = rng.standard_normal(64)
    np.testing.assert_allclose(modulate(h, sh, -np.ones(64)), np.broadcast_to(sh, h.shape), atol=0)
    sc = rng.standard_normal(64)
    np.testing.assert_allclose(modulate(h, z, sc), h + h * sc, rtol=1e-15, atol=1e-15)


def test_modulation_pins():
    check_modulate(O.modulate, O.layer_norm)


def check_gelu(gelu):
    xs = np.linspace(-8, 8, 1001)
    ref = np.array([0.5 * v * (1 + math.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3))) for v in xs])
    np.testing.assert_allclose(gelu(xs), ref, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(gelu(xs), tF.gelu(t64(xs), approximate="tanh").numpy(), rtol=1e-13, atol=1e-15)
    assert gelu(np.array([0.0]))[0] == 0.0


def test_gelu_tanh_pins():
    check_gelu(O.gelu_tanh)


def test_silu_pins():
    xs = np.linspace(-20, 20, 401)
    np.testing.assert_allclose(O.silu(xs), tF.silu(t64(xs)).numpy(), rtol=1e-14, atol=1e-300)


def check_softmax(softmax):
    rng = RNG(6)
    s = rng.standard_normal((9, 33)) * 10
    p = softmax(s, -1)
    assert np.all(np.abs(p.sum(-1) - 1) < 1e-12)
    np.testing.assert_allclose(p, torch.softmax(t64(s), -1).numpy(), rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(softmax(s + 1234.5, -1), p, rtol=1e-12, atol=1e-300)


def test_softmax_pins():
    check_softmax(O.softmax)


# ----------------------------------------------------------------------------------------
# Attention: brute force, library, special cases
# ----------------------------------------------------------------------------------------

def naive_attention_loops(q, k, v, heads):
    """Independent triple-loop attention (pure Python) for tiny inputs."""
    Lq, D = len(q), len(q[0])
    Lk = len(k)
    d = D // heads
    out = [[0.0] * D for _ in range(Lq)]
    for hh in range(heads):
        for i in range(Lq):
            scores = []
            for j in range(Lk):
                acc = 0.0
                for c in range(hh * d, (hh + 1) * d):
                    acc += q[i][c] * k[j][c]
                scores.append(acc / math.sqrt(d))
            mx = max(scores)
            ex = [math.exp(sv - mx) for sv in scores]
            den = sum(ex)
            for c in range(hh * d, (hh + 1) * d):
                out[i][c] = sum(ex[j] * v[j][c] for j in range(Lk)) / den
    return np.array(out)


def check_attention(attention):
    rng = RNG(7)
    for Lq, Lk, H, d in [(5, 7, 2, 4), (3, 1, 1, 8), (6, 13, 3, 2)]:
        q = rng.standard_normal((Lq, H * d)) * 2
        k = rng.standard_normal((Lk, H * d)) * 2
        v = rng.standard_normal((Lk, H * d))
        got = attention(q, k, v, H)
        np.testing.assert_allclose(got, naive_attention_loops(q.tolist(), k.tolist(), v.tolist(), H),
                                   rtol=1e-12, atol=1e-13)
        qt = t64(q).reshape(Lq, H, d).transpose(0, 1)
        kt = t64(k).reshape(Lk, H, d).transpose(0, 1)
        vt = t64(v).reshape(Lk, H, d).transpose(0, 1)
        ref = tF.scaled_dot_product_attention(qt, kt, vt).transpose(0, 1).reshape(Lq, H * d).numpy()
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    # one key: output is that key's value
    q = rng.standard_normal((4, 8)); k = rng.standard_normal((1, 8)); v = rng.standard_normal((1, 8))
    np.testing.assert_allclose(attention(q, k, v, 2), np.repeat(v, 4, 0), rtol=1e-14)
    # all keys equal: output is the mean of the values
    k = np.repeat(rng.standard_normal((1, 8)), 6, 0); v = rng.standard_normal((6, 8))
    np.testing.assert_allclose(attention(q, k, v, 2), np.repeat(v.mean(0, keepdims=True), 4, 0), rtol=1e-13)
    # keys/values permuted together: same output
    k = rng.standard_normal((9, 8)); v = rng.standard_normal((9, 8)); perm = rng.permutation(9)
    np.testing.assert_allclose(attention(q, k[perm], v[perm], 2), attention(q, k, v, 2), rtol=1e-12)


def test_attention_pins():
    check_attention(O.attention)


def test_attention_long_rows_chunking():
    """Query-row chunking inside the oracle (memory bound only) changes nothing."""
    rng = RNG(8)
    q = rng.standard_normal((1100, 16)); k = rng.standard_normal((40, 16)); v = rng.standard_normal((40, 16))
    full = O.attention(q, k, v, 2)
    np.testing.assert_allclose(full[1000:], O.attention(q[1000:], k, v, 2), rtol=0, atol=0)


# ----------------------------------------------------------------------------------------
# Block: library re-expression, special cases, invariants, row sampling
# ----------------------------------------------------------------------------------------

def torch_fp8_linear(t, W, b):
    """linear with E4M3 codes made by torch's float8_e4m3fn conversion: per-row scales of
    the input, one scale for the weight (scale = amax / 448 in float32)."""
    def codes(a, dim):
        a32 = a.to(torch.float32)
        amax = a32.abs().amax(dim=dim, keepdim=True) if dim is not None else a32.abs().amax()
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        return (a32 / sc).to(torch.float8_e4m3fn).to(torch.float64), sc.to(torch.float64)
    qx, sx = codes(t, -1)
    qw, sw = codes(W, None)
    return (qx @ qw.T) * sx * sw + b


def torch_block(x, e, w, ctx, heads, eps=1e-6, img_ctx=None, fp8=False, fp8_attention=False):
    """The block re-expressed with torch library routines (layer_norm, linear,
    scaled_dot_product_attention, gelu) in float64; with ``fp8`` every linear layer
    uses torch's E4M3 conversion (``torch_fp8_linear``), with ``fp8_attention`` the
    self-attention is ``torch_attention_fp8``."""
    X, E, C = t64(x), t64(e) + t64(w["mod_bias"]), t64(ctx)
    lin = torch_fp8_linear if fp8 else tF.linear
    D = X.shape[-1]
    d = D // heads
    W = {k: t64(v) for k, v in w.items()}

    def mha(q, k, v):
        Lq, Lk = q.shape[0], k.shape[0]
        qh = q.reshape(Lq, heads, d).transpose(0, 1)
        kh = k.reshape(Lk, heads, d).transpose(0, 1)
        vh = v.reshape(Lk, heads, d).transpose(0, 1)
        return tF.scaled_dot_product_attention(qh, kh, vh).transpose(0, 1).reshape(Lq, D)

    ln = lambda t: tF.layer_norm(t, (D,), eps=eps)  # noqa: E731
    h = ln(X) * (1 + E[1]) + E[0]
    qkv = lin(h, W["w_qkv"], W["b_qkv"])
    sa_in = (qkv[:, :D], qkv[:, D:2 * D], qkv[:, 2 * D:])
    o_sa = t64(torch_attention_fp8(*(a.numpy() for a in sa_in), heads)) if fp8_attention else mha(*sa_in)
    X = X + E[2] * lin(o_sa, W["w_o"], W["b_o"])
    hc = ln(X)
    q = lin(hc, W["w_cq"], W["b_cq"])
    kv = lin(C, W["w_ckv"], W["b_ckv"])
    o = mha(q, kv[:, :D], kv[:, D:])
    if img_ctx is not None:
        kvi = lin(t64(img_ctx), W["w_ckv_img"], W["b_ckv_img"])
        o = o + mha(q, kvi[:, :D], kvi[:, D:])
    X = X + lin(o, W["w_co"], W["b_co"])
    hf = ln(X) * (1 + E[4]) + E[3]
    ff = lin(tF.gelu(lin(hf, W["w_1"], W["b_1"]), approximate="tanh"), W["w_2"], W["b_2"])
    return (X + E[5] * ff).numpy()


def _tiny_block_inputs(i2v=False, seed=0):
    w = WORKLOADS["wan13b_480p_i2v_block" if i2v else "tiny_f32_block"]
    if i2v:
        import dataclasses
        w = dataclasses.replace(w, frames=2, height=4, width=8, dim=64, heads=2, ffn=96, text_len=9,
                                img_len=5, img_feat=24, dtype="f32")
    inp = make_inputs(w, seed=seed)
    return w, inp


def check_block_vs_torch(dit_block):
    for i2v in (False, True):
        w, inp = _tiny_block_inputs(i2v)
        blk = inp["blocks"][0]
        img = None
        if i2v:
            img = O.image_context_mlp(inp["img_feat"][0], inp["w_i1"], inp["b_i1"], inp["w_i2"],
                                      inp["b_i2"], inp["w_i3"], inp["b_i3"])
        got = dit_block(inp["x"][0], inp["e"][0], blk, inp["ctx"][0], w.heads, img_ctx=img)
        ref = torch_block(inp["x"][0], inp["e"][0], blk, inp["ctx"][0], w.heads, img_ctx=img)
        np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(got - inp["x"][0], ref - inp["x"][0], rtol=1e-9, atol=1e-11)


def test_block_matches_library_reexpression():
    check_block_vs_torch(O.dit_block)


def check_block_special_cases(dit_block):
    w, inp = _tiny_block_inputs()
    x, e, ctx = inp["x"][0].astype(np.float64), inp["e"][0].astype(np.float64), inp["ctx"][0]
    blk = {k: np.asarray(v, dtype=np.float64) for k, v in inp["blocks"][0].items()}
    e0 = e.copy()
    e0[2] = -blk["mod_bias"][2]          # gate_msa = 0 exactly
    e0[5] = -blk["mod_bias"][5]          # gate_ffn = 0 exactly
    out = dit_block(x, e0, blk, ctx, w.heads)
    ca = O.cross_attention_branch(O.layer_norm(x), ctx, blk, w.heads)
    np.testing.assert_allclose(out, x + ca, rtol=1e-13, atol=1e-13)
    blk0 = dict(blk, w_co=np.zeros_like(blk["w_co"]), b_co=np.zeros_like(blk["b_co"]))
    assert np.array_equal(dit_block(x, e0, blk0, ctx, w.heads), x)      # identity block
    perm = RNG(9).permutation(ctx.shape[0])                              # text order is irrelevant
    np.testing.assert_allclose(dit_block(x, e, blk, ctx[perm], w.heads), dit_block(x, e, blk, ctx, w.heads),
                               rtol=1e-12, atol=1e-12)


def test_block_gates_identity_and_text_permutation():
    check_block_special_cases(O.dit_block)


def test_block_row_sampling_is_exact():
    w, inp = _tiny_block_inputs()
    x, e, ctx, blk = inp["x"][0], inp["e"][0], inp["ctx"][0], inp["blocks"][0]
    full = O.dit_block(x, e, blk, ctx, w.heads)
    rows = [0, 5, 17, 31]
    np.testing.assert_allclose(O.dit_block(x, e, blk, ctx, w.heads, rows=rows), full[rows], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------------------
# I2V, image MLP, head, stack, flow matching
# ----------------------------------------------------------------------------------------

def check_i2v_mask(i2v_mask):
    keep = np.zeros(81); keep[0] = 1
    m = i2v_mask(keep, 21, 6, 4)
    assert m.shape == (4, 21, 6, 4)
    assert np.all(m[:, 0] == 1) and np.all(m[:, 1:] == 0)
    keep = np.zeros(81); keep[80] = 1                  # last pixel frame -> channel 3 of the last latent frame
    m = i2v_mask(keep, 21, 2, 2)
    assert m[3, 20].min() == 1 and m.sum() == 4
    keep = np.zeros(81); keep[1] = 1                   # second pixel frame -> channel 0 of latent frame 1
    m = i2v_mask(keep, 21, 2, 2)
    assert m[0, 1].min() == 1 and m.sum() == 4


def test_i2v_mask_structure():
    check_i2v_mask(O.i2v_mask)


def check_i2v_input(i2v_input):
    """With the 20 extra input channels' weights at zero (their initialisation), the
    36-channel patchify is the text-to-video one on the noise; the condition latent sits
    in channels 16-31 and the mask in 32-35."""
    rng = RNG(10)
    D, F, H, W = 12, 2, 4, 6
    noise, cond = rng.standard_normal((16, F, H, W)), rng.standard_normal((16, F, H, W))
    keep = np.zeros(1 + 4 * (F - 1)); keep[0] = 1
    mask = O.i2v_mask(keep, F, H, W)
    x36 = i2v_input(noise, cond, mask)
    assert x36.shape == (36, F, H, W)
    w16 = rng.standard_normal((D, 16, 1, 2, 2)); b = rng.standard_normal(D)
    w36 = np.concatenate([w16, np.zeros((D, 20, 1, 2, 2))], axis=1)
    assert np.array_equal(O.patchify(x36, w36, b), O.patchify(noise, w16, b))
    assert np.array_equal(x36[16:32], cond) and np.array_equal(x36[32:], mask)
    w36[:, 16:] = rng.standard_normal((D, 20, 1, 2, 2))
    assert not np.allclose(O.patchify(x36, w36, b), O.patchify(noise, w16, b))


def test_i2v_zero_projection_equals_t2v():
    check_i2v_input(O.i2v_input)


def check_image_context_mlp(mlp):
    """Linear -> GELU-tanh -> Linear -> GELU-tanh -> Linear, re-expressed in torch."""
    rng = RNG(11)
    feat = rng.standard_normal((5, 24))
    ws = [rng.standard_normal(s) * 0.2 for s in [(16, 24), (16,), (16, 16), (16,), (16, 16), (16,)]]
    ref = t64(feat)
    for i in range(3):
        ref = tF.linear(ref, t64(ws[2 * i]), t64(ws[2 * i + 1]))
        if i < 2:
            ref = tF.gelu(ref, approximate="tanh")
    np.testing.assert_allclose(mlp(feat, *ws), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_image_context_mlp_vs_torch():
    check_image_context_mlp(O.image_context_mlp)


def check_head(head):
    """Plain LayerNorm (eps 1e-6, no affine) then Linear(D, out_ch * 4), in torch."""
    rng = RNG(14)
    x = rng.standard_normal((7, 32)) * 3 + 1.5
    w, b = rng.standard_normal((64, 32)) * 0.1, rng.standard_normal(64)
    ref = tF.linear(tF.layer_norm(t64(x), (32,), eps=1e-6), t64(w), t64(b))
    np.testing.assert_allclose(head(x, w, b), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_head_vs_torch():
    check_head(O.head)


def check_stack(dit_stack):
    """All-zero blocks leave the stack as head(patchify) (in torch); two real blocks equal
    the torch re-expression of the block applied in order with the shared MLP output."""
    w = WORKLOADS["tiny_f32_block"]
    inp = make_inputs(w, seed=1, n_blocks=2)
    lat, t, ctx = inp["noise"][0], float(inp["t"][0]), inp["ctx"][0]
    zero = [{k: np.zeros_like(v) for k, v in b.items()} for b in inp["blocks"]]
    v = dit_stack(lat, t, inp, zero, ctx, w.heads)
    x = O.patchify(lat, inp["w_p"], inp["b_p"])
    ref = O.unpatchify(tF.linear(tF.layer_norm(t64(x), (w.dim,), eps=1e-6), t64(inp["w_head"]),
                                 t64(inp["b_head"])).numpy(), 16, w.frames, w.height, w.width)
    np.testing.assert_allclose(v, ref, rtol=1e-12, atol=1e-12)
    v2 = dit_stack(lat, t, inp, inp["blocks"], ctx, w.heads)
    e = O.time_mlp(t, inp["w_t1"], inp["b_t1"], inp["w_t2"], inp["b_t2"])
    xx = x
    for b in inp["blocks"]:
        xx = torch_block(xx, e, b, ctx, w.heads)
    ref2 = O.unpatchify(O.head(xx, inp["w_head"], inp["b_head"]), 16, w.frames, w.height, w.width)
    np.testing.assert_allclose(v2, ref2, rtol=1e-10, atol=1e-11)
    return inp, lat, t, ctx, x, e, v2


def test_stack_with_zero_blocks_is_head_of_patchify_and_matches_blockwise():
    w = WORKLOADS["tiny_f32_block"]
    inp, lat, t, ctx, x, e, v2 = check_stack(O.dit_stack)
    # the FP8 stack == the torch re-expression of the FP8 block (torch's E4M3 conversion)
    # applied twice; patchify, the time MLP and the head unchanged
    v3 = O.dit_stack(lat, t, inp, inp["blocks"], ctx, w.heads, fp8=True)
    xx = x
    for b in inp["blocks"]:
        xx = torch_block(xx, e, b, ctx, w.heads, fp8=True)
    ref3 = O.unpatchify(O.head(xx, inp["w_head"], inp["b_head"]), 16, w.frames, w.height, w.width)
    np.testing.assert_allclose(v3, ref3, rtol=1e-9, atol=1e-10)
    assert not np.allclose(v3, v2)


# ----------------------------------------------------------------------------------------
# The float32-product / float64-reduction stack used for the full-size 30-block stack
# ----------------------------------------------------------------------------------------

def check_attention_f32(attn_f32):
    """Against the float64 ``attention``: scores spanning several 128-key partial sums
    and a ragged tail, query blocks with a ragged last one, logit std 1 and 4."""
    rng = RNG(40)
    for scale in (1.0, 4.0):
        q = rng.standard_normal((300, 256)) * scale / 64 ** 0.25 * 1.0
        k = rng.standard_normal((300, 256)) / 64 ** 0.25
        v = rng.standard_normal((300, 256))
        got = np.asarray(attn_f32(q, k, v, 4, chunk=128))
        ref = O.attention(np.float32(q), np.float32(k), np.float32(v), 4)
        assert np.abs(got - ref).max() <= 2e-6 * np.abs(ref).max(), np.abs(got - ref).max()


def check_stack_f32(stack_f32, block_f32=None):
    """Against the float64 ``dit_stack``: a 3-block full-width stack at 144 tokens (one
    whole 128-key block plus a ragged tail), T2V and I2V, the whole velocity and the
    head outputs of sampled tokens, within 2e-6 of max|v| (float32 products)."""
    import dataclasses
    for name in ("wan13b_480p_stack30", "wan13b_480p_i2v_block"):
        w = dataclasses.replace(WORKLOADS[name], frames=3, height=12, width=16, dim=256, heads=2, ffn=512,
                                text_len=24, img_len=20 if name.endswith("i2v_block") else 0, img_feat=64,
                                n_blocks=3)
        inp = make_inputs(w, seed=3, block_input=False, zero_wx=False)
        lat = inp["noise"][0]
        img = None
        if w.i2v:
            img = round_bf16(RNG(41).standard_normal((w.img_len, w.dim)).astype(np.float32))
            lat = np.concatenate([lat, inp["cond"][0], np.zeros((4, w.frames, w.height, w.width), np.float32)])
        t = float(inp["u"][0] * 1000.0) if "u" in inp else float(inp["t"][0])
        ref = O.dit_stack(lat, t, inp, inp["blocks"], inp["ctx"][0], w.heads, img_ctx=img)
        got = stack_f32(lat, t, inp, inp["blocks"], inp["ctx"][0], w.heads, img_ctx=img)
        den = np.abs(ref).max()
        assert np.abs(got - ref).max() <= 2e-6 * den, (name, np.abs(got - ref).max() / den)
        rows = np.array([0, 7, 100, 127, 128, 143])
        y = np.asarray(ref).reshape(16, w.frames, w.height // 2, 2, w.width // 2, 2)
        y = y.transpose(1, 2, 4, 0, 3, 5).reshape(w.tokens, 64)
        got_rows = stack_f32(lat, t, inp, inp["blocks"], inp["ctx"][0], w.heads, img_ctx=img, rows=rows)
        assert np.abs(got_rows - y[rows]).max() <= 2e-6 * den


def test_attention_f32_matches_float64_attention():
    check_attention_f32(O.attention_f32)


def test_stack_f32_matches_float64_stack():
    check_stack_f32(O.dit_stack_f32)


def check_flow_matching(fm_input, fm_target):
    """x_t runs from x0 at t = 0 to x1 at t = 1 on a straight line whose velocity is the
    target: x_0.75 - x_0.25 = 0.5 v."""
    rng = RNG(12)
    x1, x0 = rng.standard_normal((3, 4)), rng.standard_normal((3, 4))
    assert np.array_equal(fm_input(x1, x0, 0.0), x0)
    assert np.array_equal(fm_input(x1, x0, 1.0), x1)
    a, b = fm_input(x1, x0, 0.25), fm_input(x1, x0, 0.75)
    np.testing.assert_allclose(b - a, 0.5 * fm_target(x1, x0), rtol=1e-14, atol=1e-15)


def test_flow_matching_endpoints():
    check_flow_matching(O.flow_matching_input, O.flow_matching_target)


# ----------------------------------------------------------------------------------------
# Input generator (shared with the CUDA tests): bf16 rounding and row sampling
# ----------------------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = RNG(13)
    a = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.4e38, -1e-40], np.float32)])
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits(a), ref)
    assert np.array_equal(round_bf16(a), torch.from_numpy(a).to(torch.bfloat16).float().numpy())
    assert np.array_equal(bits_to_f32(bf16_bits(a)), round_bf16(a))


def test_sample_rows_cover_ends_and_ragged_tail():
    rows = sample_rows(32760)
    assert len(rows) == 256 and rows[0] == 0 and rows[-1] == 32759
    assert set(range(32640, 32760)).issubset(set(rows.tolist()))
    assert np.array_equal(sample_rows(100), np.arange(100))


def test_inputs_are_deterministic():
    w = WORKLOADS["tiny_f32_block"]
    a, b = make_inputs(w, seed=0), make_inputs(w, seed=0)
    assert np.array_equal(a["x"], b["x"]) and np.array_equal(a["blocks"][0]["w_qkv"], b["blocks"][0]["w_qkv"])
    assert not np.array_equal(a["x"], make_inputs(w, seed=1)["x"])


# ----------------------------------------------------------------------------------------
# Sampling loop: Euler integration with classifier-free guidance
# ----------------------------------------------------------------------------------------

def check_euler_cfg(euler_cfg):
    rng = RNG(14)
    x0 = rng.standard_normal((3, 4))
    c = rng.standard_normal((3, 4))
    u = rng.standard_normal((3, 4))
    # constant velocities: x(1) = x0 + u + g (c - u), for any step count
    for n in (1, 3, 50):
        for g in (0.0, 1.0, 5.0):
            got = euler_cfg(x0, n, g, lambda x, t: c, lambda x, t: u)
            np.testing.assert_allclose(got, x0 + u + g * (c - u), rtol=1e-12, atol=1e-12)
    # linear ODE dx/dt = a x: Euler gives (1 + a/n)^n x0 exactly
    a = -0.7
    for n in (1, 4, 50):
        got = euler_cfg(x0, n, 1.0, lambda x, t: a * x, lambda x, t: 0 * x)
        np.testing.assert_allclose(got, (1 + a / n) ** n * x0, rtol=1e-12)
    # time-dependent velocity v = t: Euler on the left grid gives sum_k k/n^2 = (n-1)/(2n)
    for n in (1, 2, 10):
        got = euler_cfg(x0, n, 1.0, lambda x, t: np.full_like(x, t), lambda x, t: 0 * x)
        np.testing.assert_allclose(got, x0 + (n - 1) / (2 * n), rtol=1e-12)


def test_euler_cfg_closed_forms():
    check_euler_cfg(O.euler_cfg)


def test_sampler_uses_stack_velocity():
    """One step with guidance 1 is x0 + v_cond(x0, t=0); guidance 0 uses the
    unconditional context only."""
    w = WORKLOADS["tiny_f32_block"]
    inp = make_inputs(w, seed=2, n_blocks=1)
    x0 = inp["noise"][0]
    ctx_c, ctx_u = inp["ctx"][0], RNG(15).standard_normal(inp["ctx"][0].shape)
    v_c = O.dit_stack(x0, 0.0, inp, inp["blocks"], ctx_c, w.heads)
    v_u = O.dit_stack(x0, 0.0, inp, inp["blocks"], ctx_u, w.heads)
    got1 = O.sample_euler_cfg(x0, 1, 1.0, inp, inp["blocks"], ctx_c, ctx_u, w.heads)
    np.testing.assert_allclose(got1, x0 + v_c, rtol=1e-12, atol=1e-12)
    got0 = O.sample_euler_cfg(x0, 1, 0.0, inp, inp["blocks"], ctx_c, ctx_u, w.heads)
    np.testing.assert_allclose(got0, x0 + v_u, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ diffusion cache
def check_cache_schedule(schedule_fn):
    s = schedule_fn(10, 2, 3, 5, 2)
    assert [k for k, (ra, _) in enumerate(s) if ra] == [3, 4, 6, 7, 9]
    assert [k for k, (_, su) in enumerate(s) if su] == [6, 8]
    assert not any(ra or su for ra, su in schedule_fn(6, 0, 1, 0, 1))       # interval 1: never reuse
    assert not any(ra or su for ra, su in schedule_fn(4, 4, 2, 9, 2))       # starts past the end
    assert schedule_fn(3, 0, 2, 1, 5) == [(False, False), (True, False), (False, True)]


def test_cache_schedule_closed_forms():
    check_cache_schedule(O.diffusion_cache_schedule)


def check_euler_cfg_cached(euler_cfg_cached):
    rng = RNG(16)
    x0 = rng.standard_normal((3, 4))
    c, u = rng.standard_normal((3, 4)), rng.standard_normal((3, 4))
    never = [(False, False)] * 5
    # no caching: the uncached loop, bitwise
    fc = lambda x, t, r: 0.3 * x + t * c                                     # noqa: E731
    fu = lambda x, t, r: -0.2 * x + u                                        # noqa: E731
    ref = O.euler_cfg(x0, 5, 4.0, lambda x, t: fc(x, t, False), lambda x, t: fu(x, t, False))
    assert np.array_equal(euler_cfg_cached(x0, 5, 4.0, fc, fu, never), ref)
    # constant velocities: the kept difference is exact, any schedule gives x0 + u + g (c - u)
    sched = [(False, False), (True, True), (True, False), (False, True), (True, True)]
    got = euler_cfg_cached(x0, 5, 5.0, lambda x, t, r: c, lambda x, t, r: u, sched)
    np.testing.assert_allclose(got, x0 + u + 5.0 * (c - u), rtol=1e-12, atol=1e-12)
    # linear velocities a x, b x, two steps, the second skips the unconditional pass:
    # x1 = x0 + (b + g (a - b)) x0 / 2, x2 = x1 + (a x1 + (g - 1)(a - b) x0) / 2
    a, b, g = 0.7, -0.4, 3.0
    got = euler_cfg_cached(x0, 2, g, lambda x, t, r: a * x, lambda x, t, r: b * x, [(False, False), (False, True)])
    x1 = x0 + 0.5 * (b + g * (a - b)) * x0
    np.testing.assert_allclose(got, x1 + 0.5 * (a * x1 + (g - 1) * (a - b) * x0), rtol=1e-12)
    # the reuse flag of each step reaches both velocity calls; skipped steps call v_u not at all
    seen = []
    euler_cfg_cached(x0, 3, 2.0, lambda x, t, r: seen.append(("c", t, r)) or c,
                     lambda x, t, r: seen.append(("u", t, r)) or u, [(False, False), (True, True), (True, False)])
    assert seen == [("c", 0.0, False), ("u", 0.0, False), ("c", 1 / 3, True), ("c", 2 / 3, True), ("u", 2 / 3, True)]


def test_euler_cfg_cached_closed_forms():
    check_euler_cfg_cached(O.euler_cfg_cached)


def check_block_attention_cache(dit_block):
    w, inp = _tiny_block_inputs(seed=3)
    x, e, blk, ctx = inp["x"][0], inp["e"][0], inp["blocks"][0], inp["ctx"][0]
    cache = {}
    y0 = dit_block(x, e, blk, ctx, w.heads, attn_cache=cache)
    o0 = cache["o"].copy()
    # same input, reuse: identical output, cache untouched
    cache["reuse"] = True
    assert np.array_equal(dit_block(x, e, blk, ctx, w.heads, attn_cache=cache), y0)
    assert np.array_equal(cache["o"], o0)
    # a new input with reuse keeps the old attention output o0 (then the output
    # projection, gate, cross-attention and FFN of the new input)
    x2 = x + 0.3 * RNG(17).standard_normal(x.shape)
    got = dit_block(x2, e, blk, ctx, w.heads, attn_cache=cache)
    mod = O.block_modulation(e, blk["mod_bias"])
    x1 = x2 + mod[2] * (o0 @ blk["w_o"].astype(np.float64).T + blk["b_o"])
    x2b = x1 + O.cross_attention_branch(O.layer_norm(x1), ctx, blk, w.heads)
    want = x2b + mod[5] * O.ffn_branch(O.modulate(O.layer_norm(x2b), mod[3], mod[4]), blk)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    assert not np.allclose(got, dit_block(x2, e, blk, ctx, w.heads))           # reuse did change the result
    # recomputing on the new input refreshes the cache and equals the plain block
    cache["reuse"] = False
    np.testing.assert_allclose(dit_block(x2, e, blk, ctx, w.heads, attn_cache=cache),
                               dit_block(x2, e, blk, ctx, w.heads), rtol=1e-12, atol=1e-12)
    assert not np.allclose(cache["o"], o0)


def test_block_attention_cache():
    check_block_attention_cache(O.dit_block)


def test_cached_sampler_without_reuse_is_the_sampler():
    w = WORKLOADS["tiny_f32_block"]
    inp = make_inputs(w, seed=4, n_blocks=2)
    x0 = inp["noise"][0]
    ctx_c, ctx_u = inp["ctx"][0], RNG(18).standard_normal(inp["ctx"][0].shape)
    sched = O.diffusion_cache_schedule(3, 0, 1, 0, 1)
    got = O.sample_euler_cfg_cached(x0, 3, 4.0, inp, inp["blocks"], ctx_c, ctx_u, w.heads, sched)
    assert np.array_equal(got, O.sample_euler_cfg(x0, 3, 4.0, inp, inp["blocks"], ctx_c, ctx_u, w.heads))
    # with reuse the result moves, but stays close (the cache is an approximation)
    sched = O.diffusion_cache_schedule(3, 1, 2, 2, 2)
    assert sched == [(False, False), (False, False), (True, False)]
    got2 = O.sample_euler_cfg_cached(x0, 3, 4.0, inp, inp["blocks"], ctx_c, ctx_u, w.heads, sched)
    assert not np.array_equal(got2, got)


# ------------------------------------------------------------------ FP8 (E4M3)
def check_e4m3_decode(decode):
    assert decode(0x7E) == 448.0 and decode(0x38) == 1.0 and decode(0x08) == 2.0 ** -6
    assert decode(0x01) == 2.0 ** -9 and decode(0x00) == 0.0 and decode(0x3C) == 1.5
    assert math.isnan(decode(0x7F)) and math.isnan(decode(0xFF))
    vals = [decode(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))                     # monotone in code order
    assert all(decode(c | 0x80) == -decode(c) for c in range(0x7F))


def test_e4m3_decode_closed_forms():
    check_e4m3_decode(O.e4m3_decode)


def check_round_e4m3(round_fn):
    vals = np.array([O.e4m3_decode(c) for c in range(0x7F)])
    assert np.array_equal(round_fn(vals), vals) and np.array_equal(round_fn(-vals), -vals)   # fixed points
    mids = (vals[:-1] + vals[1:]) / 2                                        # ties go to the even code
    got = round_fn(mids)
    even = np.where(np.arange(len(mids)) % 2 == 0, vals[:-1], vals[1:])
    assert np.array_equal(got, even)
    x = RNG(19).uniform(-448, 448, 20000) * np.exp2(RNG(20).integers(-14, 1, 20000))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(round_fn(x), ref)                                  # library conversion, in range
    assert np.array_equal(round_fn(np.array([449.0, 1e6, -500.0])), np.array([448.0, 448.0, -448.0]))


def test_round_e4m3_grid_ties_and_library():
    check_round_e4m3(O.round_e4m3)


def test_quantize_e4m3_scales():
    a = RNG(21).standard_normal((7, 33)) * np.exp2(RNG(22).integers(-8, 8, (7, 1)))
    a[3] = 0.0
    q, s = O.quantize_e4m3(a, axis=-1)
    assert s.shape == (7, 1) and s[3, 0] == 1.0 and not q[3].any()
    rows = [r for r in range(7) if r != 3]
    assert np.all(np.abs(q[rows]).max(axis=1) == 448.0)                     # the row max maps to 448
    err = np.abs(q * s.astype(np.float64) - a)
    assert np.all(err <= 2.0 ** -4 * np.abs(a) + s.astype(np.float64) * 2.0 ** -10 + 1e-30)
    qt, st = O.quantize_e4m3(a)
    assert np.ndim(st) == 0 and np.abs(qt).max() == 448.0


def test_linear_fp8_is_the_dequantised_product():
    r = RNG(23)
    x, w, b = r.standard_normal((9, 40)), 0.02 * r.standard_normal((24, 40)), r.standard_normal(24)
    qx, sx = O.quantize_e4m3(x, axis=-1)
    qw, sw = O.quantize_e4m3(w)
    ref = O.linear(qx * sx.astype(np.float64), qw * np.float64(sw), b)
    np.testing.assert_allclose(O.linear_fp8(x, w, b), ref, rtol=1e-12, atol=1e-12)
    exact = O.linear(x, w, b) - b
    assert np.abs(O.linear_fp8(x, w, b) - b - exact).max() < 0.1 * np.abs(exact).max()   # an approximation of it


def check_block_fp8_vs_torch(dit_block):
    for i2v, fa in ((False, False), (True, False), (False, True), (True, True)):
        w, inp = _tiny_block_inputs(i2v, seed=6)
        blk = inp["blocks"][0]
        img = None
        if i2v:
            img = O.image_context_mlp(inp["img_feat"][0], inp["w_i1"], inp["b_i1"], inp["w_i2"],
                                      inp["b_i2"], inp["w_i3"], inp["b_i3"])
        got = dit_block(inp["x"][0], inp["e"][0], blk, inp["ctx"][0], w.heads, img_ctx=img, fp8=True,
                        fp8_attention=fa)
        ref = torch_block(inp["x"][0], inp["e"][0], blk, inp["ctx"][0], w.heads, img_ctx=img, fp8=True,
                          fp8_attention=fa)
        np.testing.assert_allclose(got - inp["x"][0], ref - inp["x"][0], rtol=1e-9, atol=1e-10)
        plain = dit_block(inp["x"][0], inp["e"][0], blk, inp["ctx"][0], w.heads, img_ctx=img)
        d, dp = got - inp["x"][0], plain - inp["x"][0]
        assert 0 < np.abs(d - dp).max() < 0.2 * np.abs(dp).max()             # close to, not equal to, bf16


def test_block_fp8_matches_library_reexpression():
    check_block_fp8_vs_torch(O.dit_block)


# ----------------------------------------------------------------------------------------
# 8-bit attention
# ----------------------------------------------------------------------------------------

def torch_attention_fp8(q, k, v, heads):
    """The same definition through torch's float8_e4m3fn conversion (float32 scales and
    divisions, as in the kernels' quantisers)."""
    q, k, v = (torch.from_numpy(np.asarray(a, dtype=np.float32)) for a in (q, k, v))
    d = q.shape[1] // heads
    f8 = torch.float8_e4m3fn

    def scale(a, dim=None):
        m = a.abs().amax(dim=dim, keepdim=dim is not None)
        return torch.where(m > 0, m / 448.0, torch.ones_like(m))
    outs = []
    for h in range(heads):
        qh, kh, vh = (a[:, h * d:(h + 1) * d] for a in (q, k, v))
        sq, sk, sv = scale(qh, 1), scale(kh), scale(vh)
        qc, kc, vc = ((a / s).to(f8).double() for a, s in ((qh, sq), (kh, sk), (vh, sv)))
        x = (qc @ kc.T) * sq.double() * sk.double() / math.sqrt(d) / math.log(2.0)
        p = torch.exp2(x - torch.ceil(x.amax(1, keepdim=True)))
        outs.append(sv.double() * (p.to(f8).double() @ vc) / p.sum(1, keepdim=True))
    return torch.cat(outs, 1).numpy()


def check_attention_fp8(attention_fp8):
    rng = RNG(31)
    for Lq, Lk, H, d in [(5, 7, 2, 16), (9, 40, 3, 8), (4, 1, 1, 32)]:
        q = rng.standard_normal((Lq, H * d)) * np.exp2(rng.integers(-3, 4, (Lq, 1)))
        k = rng.standard_normal((Lk, H * d)) * 2
        v = rng.standard_normal((Lk, H * d))
        got = attention_fp8(q, k, v, H)
        np.testing.assert_allclose(got, torch_attention_fp8(q, k, v, H), rtol=1e-12, atol=1e-13)
        exact = O.attention(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32), H)
        assert np.abs(got - exact).max() < 0.15 * np.abs(exact).max()        # an approximation of it
    # values on the E4M3 grid with a power-of-two scale are represented exactly, and a
    # zero query makes every logit 0, so p = 1 exactly: one key gives that key's value,
    # several keys the mean of the values
    grid = np.array([O.e4m3_decode(c) for c in range(0x7F)])
    v = rng.choice(grid, (6, 16)) * rng.choice([-1.0, 1.0], (6, 16)) / 16.0
    v[0, 0] = 448.0 / 16.0                                                   # scale 2^-4 for both heads
    v[0, 8] = -448.0 / 16.0
    q0 = np.zeros((4, 16))
    np.testing.assert_array_equal(attention_fp8(q0, rng.standard_normal((1, 16)), v[:1], 2), np.repeat(v[:1], 4, 0))
    np.testing.assert_allclose(attention_fp8(q0, rng.standard_normal((6, 16)), v, 2),
                               np.repeat(v.mean(0, keepdims=True), 4, 0), rtol=1e-15, atol=1e-15)
    q = rng.standard_normal((4, 16))
    # keys and values permuted together: same output
    k, v = rng.standard_normal((11, 16)), rng.standard_normal((11, 16))
    perm = rng.permutation(11)
    np.testing.assert_allclose(attention_fp8(q, k[perm], v[perm], 2), attention_fp8(q, k, v, 2), rtol=1e-12)


def test_attention_fp8_pins():
    check_attention_fp8(O.attention_fp8)


def check_attention_fp8_running_base(attn):
    """The running-base option of ``attention_fp8`` (the base a one-pass kernel keeps).

    (1) Where every p stays in E4M3's normal range under both bases, the codes differ
    only by exact powers of two, so the option equals the definition (whole and with
    key-split query blocks) to rounding of float64 sums.
    (2) A hand-built case whose base trajectory is known: one head (d = 128), keys in two
    128-key tiles. Every query and key has one non-zero component, so logit (log2 units)
    = alpha_r * k_j with k on the E4M3 grid (k scale 1/16). Tile 0: all k = 0 (p = 1 for
    every row). Tile 1: a jump key k = 28, a key k = -20 whose value is e_0, and k = 0
    elsewhere; key 0 (tile 0) has value e_1; the other values are zero.
    Row 0 (alpha 0.5) jumps by 14 > 8 in tile 1, so its warp (rows 0-31) moves: row 1
    (alpha 0.23, own jump 6.44 < 8) takes base ceil(6.44) = 7 and its p for the k = -20
    key, 2^(-4.6 - 7), rounds to zero: out[1, 0] = 0. Row 32 (the same alpha, the next
    warp, where nothing jumps; likewise row 160) keeps base 0, so that p is 2^-4.6 -> 11 * 2^-8:
    out[32, 0] = 11 * 2^-8 / l with l = 254 + 2^6.44 + 2^-4.6. Row 0 moved to base 14, so
    its tile-0 sum is scaled by 2^-14: out[0, 1] = 2^-14 / (1 + 254 * 2^-14 + 2^-24).
    With the query block split in two key halves (tile 0 | tile 1), row 32's second
    half starts at base 7: out[32, 0] = out[160, 0] = 0 and out[32, 1] = 2^-7 / (2^-7 * 128 + l1),
    l1 = 2^(6.44 - 7) + 126 * 2^-7 + 2^(-4.6 - 7)."""
    rng = RNG(52)
    for std, Lq, Lk, H in [(0.3, 300, 900, 2), (0.25, 70, 2100, 1)]:
        q = round_bf16(rng.standard_normal((Lq, H * 128)) * math.sqrt(std))
        k = round_bf16(rng.standard_normal((Lk, H * 128)) * math.sqrt(std))
        v = round_bf16(rng.standard_normal((Lk, H * 128)))
        ref = O.attention_fp8(q, k, v, H)
        for split in ((), [(0, 0)], [(h, b) for h in range(H) for b in range((Lq + 255) // 256)]):
            got = attn(q, k, v, H, running_base=True, split_units=split)
            assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max(), split
    a = math.sqrt(128) * math.log(2.0)
    q = np.zeros((192, 128))
    q[0, 0], q[1, 0], q[32, 0], q[160, 0] = 0.5 * a, 0.23 * a, 0.23 * a, 0.23 * a
    k = np.zeros((256, 128))
    k[128, 0], k[129, 0] = 28.0, -20.0
    v = np.zeros((256, 128))
    v[129, 0], v[0, 1] = 1.0, 1.0
    out = attn(q, k, v, 1, running_base=True)
    l32 = 254 + 2 ** 6.44 + 2 ** -4.6
    assert out[1, 0] == 0.0
    np.testing.assert_allclose(out[32, 0], 11 * 2.0 ** -8 / l32, rtol=1e-6)
    np.testing.assert_allclose(out[0, 1], 2.0 ** -14 / (1 + 254 * 2.0 ** -14 + 2.0 ** -24), rtol=1e-6)
    out = attn(q, k, v, 1, running_base=True, split_units=[(0, 0)])
    l1 = 2 ** (6.44 - 7) + 126 * 2.0 ** -7 + 2 ** (-4.6 - 7)
    assert out[32, 0] == 0.0 and out[160, 0] == 0.0          # row 160 is in the same 256-row block
    np.testing.assert_allclose(out[32, 1], 2.0 ** -7 / (2.0 ** -7 * 128 + l1), rtol=1e-6)
    # the definition (final row maximum) gives zero for both rows' k = -20 key
    ref = O.attention_fp8(q, k, v, 1)
    assert ref[1, 0] == 0.0 and ref[32, 0] == 0.0
    # a subset of rows is the same as those rows of the whole result
    rows = np.array([0, 1, 33, 160, 191])
    sub = attn(q, k, v, 1, running_base=True, split_units=[(0, 0)], rows=rows)
    np.testing.assert_array_equal(sub, out[rows])


def test_attention_fp8_running_base_pins():
    check_attention_fp8_running_base(O.attention_fp8)
