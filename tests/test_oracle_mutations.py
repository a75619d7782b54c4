"""Plant plausible mistakes in the oracle (on the CPU) and show the pins catch them:
a dropped term, a wrong sign or index, a transposed operand, a wrong constant."""
import math

import numpy as np
import pytest

from oracle import wan_oracle as O
import test_oracle_pins as P


def _fails(check, *args):
    with pytest.raises(AssertionError):
        check(*args)


def test_patchify_mutations_are_caught():
    def swapped_ph_pw(latent, weight, bias):          # patch flattened (pw, ph) instead of (ph, pw)
        w = np.asarray(weight).transpose(0, 1, 2, 4, 3)
        return O.patchify(latent, w, bias)

    def no_bias(latent, weight, bias):
        return O.patchify(latent, weight, np.zeros_like(bias))
    _fails(P.check_patchify, swapped_ph_pw)
    _fails(P.check_patchify, no_bias)

    def transposed_tokens(tokens, c, f, h, w):         # (j, i) token order in the inverse
        y = np.asarray(tokens).reshape(f, h // 2, w // 2, -1).transpose(0, 2, 1, 3).reshape(len(tokens), -1)
        return O.unpatchify(y, c, f, h, w)
    _fails(P.check_patch_roundtrip, O.patchify, transposed_tokens)


def test_embedding_mutations_are_caught():
    def sin_first(t, dim=256):
        e = O.sinusoidal_embedding(t, dim)
        return np.concatenate([e[dim // 2:], e[:dim // 2]])

    def wrong_base(t, dim=256):
        half = dim // 2
        a = t * np.power(1000.0, -np.arange(half) / half)
        return np.concatenate([np.cos(a), np.sin(a)])
    _fails(P.check_sinusoid, sin_first)
    _fails(P.check_sinusoid, wrong_base)

    def relu_mlp(t, w1, b1, w2, b2, freq_dim=256):
        e = O.sinusoidal_embedding(t, freq_dim)
        return O.linear(np.maximum(O.linear(e, w1, b1), 0), w2, b2).reshape(6, -1)
    _fails(P.check_time_mlp, relu_mlp, O.block_modulation)
    _fails(P.check_time_mlp, O.time_mlp, lambda e, b: np.asarray(e) + 0.5 * np.asarray(b))


def test_norm_and_activation_mutations_are_caught():
    def unbiased_ln(x, eps=1e-6):
        x = np.asarray(x, np.float64)
        return (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, ddof=1, keepdims=True) + eps)

    def eps_outside(x, eps=1e-6):
        x = np.asarray(x, np.float64)
        return (x - x.mean(-1, keepdims=True)) / (np.sqrt(x.var(-1, keepdims=True)) + eps)
    _fails(P.check_layer_norm, unbiased_ln)
    _fails(P.check_layer_norm, eps_outside)
    _fails(P.check_modulate, lambda h, sh, sc: np.asarray(h) * np.asarray(sc) + sh, O.layer_norm)
    _fails(P.check_modulate, lambda h, sh, sc: np.asarray(h) * (1 + np.asarray(sc)) - sh, O.layer_norm)

    def erf_gelu(x):
        x = np.asarray(x, np.float64)
        return np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in x])
    _fails(P.check_gelu, erf_gelu)
    _fails(P.check_gelu, lambda x: 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.0447 * x ** 3))))
    _fails(P.check_softmax, lambda s, axis=-1: np.exp(s) / np.exp(s).sum(axis, keepdims=True) * 1.0000001)


def test_attention_mutations_are_caught():
    def unscaled(q, k, v, heads):
        return O.attention(np.asarray(q) * math.sqrt(np.asarray(q).shape[1] // heads), k, v, heads)

    def heads_interleaved(q, k, v, heads):            # head h takes columns h, h+H, ... instead of a slab
        q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
        D = q.shape[1]
        perm = np.arange(D).reshape(D // heads, heads).T.reshape(-1)
        inv = np.argsort(perm)
        return O.attention(q[:, perm], k[:, perm], v[:, perm], heads)[:, inv]

    def softmax_over_queries(q, k, v, heads):
        q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
        d = q.shape[1] // heads
        out = np.empty((q.shape[0], q.shape[1]))
        for hh in range(heads):
            sl = slice(hh * d, (hh + 1) * d)
            p = O.softmax(q[:, sl] @ k[:, sl].T / math.sqrt(d), axis=0)
            out[:, sl] = p @ v[:, sl]
        return out
    _fails(P.check_attention, unscaled)
    _fails(P.check_attention, heads_interleaved)
    _fails(P.check_attention, softmax_over_queries)


def test_block_mutations_are_caught(monkeypatch):
    # gate applied to the cross-attention branch as well (wrong reading of the six vectors)
    orig = O.cross_attention_branch

    def gated_cross(h, ctx, w, heads, img_ctx=None, fp8=False):
        return 0.5 * orig(h, ctx, w, heads, img_ctx=img_ctx, fp8=fp8)
    monkeypatch.setattr(O, "cross_attention_branch", gated_cross)
    _fails(P.check_block_vs_torch, O.dit_block)
    monkeypatch.undo()

    # shift and scale rows swapped in the modulation
    orig_mod = O.block_modulation

    def swapped(e, b):
        m = orig_mod(e, b)
        return m[[1, 0, 2, 4, 3, 5]]
    monkeypatch.setattr(O, "block_modulation", swapped)
    _fails(P.check_block_vs_torch, O.dit_block)
    monkeypatch.undo()

    # FFN with the activation dropped
    monkeypatch.setattr(O, "gelu_tanh", lambda x: np.asarray(x, np.float64))
    _fails(P.check_block_vs_torch, O.dit_block)
    monkeypatch.undo()

    # image-context attention subtracted instead of added (I2V)
    orig_attn = O.attention
    calls = {"n": 0}

    def sign_flip_second(q, k, v, heads):
        calls["n"] += 1
        r = orig_attn(q, k, v, heads)
        return -r if k.shape[0] == 5 else r           # the tiny I2V image context has 5 tokens
    monkeypatch.setattr(O, "attention", sign_flip_second)
    _fails(P.check_block_vs_torch, O.dit_block)
    monkeypatch.undo()


def test_i2v_mask_mutation_is_caught():
    def no_repeat(keep, F, H, W, stride=4):
        m = np.concatenate([np.asarray(keep, np.float64), np.zeros(3)]).reshape(F, stride).T
        return np.broadcast_to(m[:, :, None, None], (stride, F, H, W)).copy()
    _fails(P.check_i2v_mask, no_repeat)


def test_euler_cfg_mutations_are_caught():
    def guidance_on_wrong_branch(x0, n, g, vc, vu):
        return O.euler_cfg(x0, n, g, vu, vc)

    def right_endpoint_grid(x0, n, g, vc, vu):
        x = np.asarray(x0, np.float64).copy()
        for k in range(n):
            t = (k + 1) / n
            x = x + (vu(x, t) + g * (vc(x, t) - vu(x, t))) / n
        return x
    _fails(P.check_euler_cfg, guidance_on_wrong_branch)
    _fails(P.check_euler_cfg, right_endpoint_grid)


def test_diffusion_cache_mutations_are_caught(monkeypatch):
    def unshifted(n, a0, ai, c0, ci):                 # period counted from step 0, not from the start
        return [(k >= a0 and k % ai != 0, k >= c0 and k % ci != 0) for k in range(n)]
    _fails(P.check_cache_schedule, unshifted)

    def flipped_residual(x0, n, g, vc, vu, sched):    # v_c - (g - 1) delta
        x = np.asarray(x0, np.float64).copy()
        delta = None
        for k in range(n):
            reuse, skip = sched[k]
            c = vc(x, k / n, reuse)
            if skip:
                v = c - (g - 1) * delta
            else:
                u = vu(x, k / n, reuse)
                delta = c - u
                v = u + g * delta
            x = x + v / n
        return x

    def stale_residual(x0, n, g, vc, vu, sched):      # delta from the first step only
        x = np.asarray(x0, np.float64).copy()
        delta = None
        for k in range(n):
            reuse, skip = sched[k]
            c = vc(x, k / n, reuse)
            if skip:
                v = c + (g - 1) * delta
            else:
                u = vu(x, k / n, reuse)
                delta = c - u if delta is None else delta
                v = u + g * (c - u)
            x = x + v / n
        return x
    _fails(P.check_euler_cfg_cached, flipped_residual)
    _fails(P.check_euler_cfg_cached, stale_residual)

    orig = O.dit_block

    def ignores_cache(x, e, w, ctx, heads, eps=1e-6, img_ctx=None, rows=None, return_parts=False, attn_cache=None):
        if attn_cache is not None and not attn_cache.get("reuse"):
            attn_cache["o"] = O.self_attention_core(O.modulate(O.layer_norm(x, eps), *O.block_modulation(
                e, w["mod_bias"])[:2]), w, heads)
        return orig(x, e, w, ctx, heads, eps, img_ctx, rows, return_parts)
    _fails(P.check_block_attention_cache, ignores_cache)


def test_fp8_mutations_are_caught(monkeypatch):
    def ties_away(x):                                  # round half away from zero instead of to even
        x = np.asarray(x, np.float64)
        a = np.abs(x)
        e = np.clip(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6, 8)
        q = np.exp2(e - 3)
        return np.sign(x) * np.minimum(np.floor(a / q + 0.5) * q, 448.0)

    def no_subnormals(x):                              # flush below 2^-6
        r = O.round_e4m3(x)
        return np.where(np.abs(np.asarray(x)) < 2.0 ** -6, 0.0, r)
    _fails(P.check_round_e4m3, ties_away)
    _fails(P.check_round_e4m3, no_subnormals)
    _fails(P.check_e4m3_decode, lambda c: O.e4m3_decode(c) * (2.0 if (c >> 3) & 0xF == 0 else 1.0))

    orig = O.quantize_e4m3

    def tensor_scales(x, axis=None):                   # one scale for all tokens instead of one per token
        q, s = orig(x)
        return (q, np.full((np.asarray(x).shape[0], 1), s, np.float32)) if axis == -1 else (q, s)
    monkeypatch.setattr(O, "quantize_e4m3", tensor_scales)
    _fails(P.check_block_fp8_vs_torch, O.dit_block)
    monkeypatch.undo()


def _attention_fp8_variant(q_axis=-1, round_p=True, norm_rounded=False, v_axis=None, int_base=True):
    def f(q, k, v, heads):
        q, k, v = (np.asarray(a, dtype=np.float32) for a in (q, k, v))
        d = q.shape[1] // heads
        out = np.empty(q.shape)
        for hh in range(heads):
            sl = slice(hh * d, (hh + 1) * d)
            qq, sq = O.quantize_e4m3(q[:, sl], axis=q_axis)
            kq, sk = O.quantize_e4m3(k[:, sl])
            vq, sv = O.quantize_e4m3(v[:, sl], axis=v_axis)
            x = (qq @ kq.T) * np.asarray(sq, np.float64) * np.float64(sk) / (math.sqrt(d) * math.log(2.0))
            m = x.max(axis=-1, keepdims=True)
            p = np.exp2(x - (np.ceil(m) if int_base else m))
            pr = O.round_e4m3(p) if round_p else p
            vv = vq * np.asarray(sv, np.float64)
            out[:, sl] = (pr @ vv) / (pr if norm_rounded else p).sum(axis=-1, keepdims=True)
        return out
    return f


def test_attention_fp8_mutations_are_caught():
    _fails(P.check_attention_fp8, _attention_fp8_variant(q_axis=None))          # one q scale per head
    _fails(P.check_attention_fp8, _attention_fp8_variant(round_p=False))        # p kept exact
    _fails(P.check_attention_fp8, _attention_fp8_variant(norm_rounded=True))    # normaliser from rounded p
    _fails(P.check_attention_fp8, _attention_fp8_variant(v_axis=-1))            # a v scale per key row
    _fails(P.check_attention_fp8, _attention_fp8_variant(int_base=False))       # base at the row max itself
    P.check_attention_fp8(_attention_fp8_variant())                              # the unmutated restatement passes


def test_f32_stack_mutations_are_caught():
    import torch

    def no_tail_sum(q, k, v, heads, chunk=2048):       # row sum misses the keys past the last 128-key block
        q32, k32, v32 = (torch.as_tensor(np.float32(a)) for a in (q, k, v))
        d = q32.shape[1] // heads
        out = np.empty(q32.shape)
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            s = q32[:, sl] @ k32[:, sl].T
            p = torch.exp((s - s.amax(-1, keepdim=True)) / math.sqrt(d))
            nb = s.shape[1] // 128
            l = p[:, :nb * 128].sum(-1, keepdim=True).double()
            out[:, sl] = ((p @ v32[:, sl]).double() / l).numpy()
        return out

    def scaled_after_exp(q, k, v, heads, chunk=2048):  # 1/sqrt(d) applied to the output, not the logits
        return np.asarray(O.attention_f32(np.asarray(q) * math.sqrt(np.asarray(q).shape[1] // heads), k, v,
                                          heads, chunk))
    _fails(P.check_attention_f32, no_tail_sum)
    _fails(P.check_attention_f32, scaled_after_exp)

    def ungated_ffn(latent, t, weights, blocks, ctx, heads, eps=1e-6, img_ctx=None, rows=None):
        mut = [dict(b) for b in blocks]
        for b in mut:                                   # gate_ffn bias zeroed: the gate is e only
            b["mod_bias"] = np.asarray(b["mod_bias"]).copy()
            b["mod_bias"][5] = 0.0
        return O.dit_stack_f32(latent, t, weights, mut, ctx, heads, eps, img_ctx=img_ctx, rows=rows)

    def last_block_all_rows(latent, t, weights, blocks, ctx, heads, eps=1e-6, img_ctx=None, rows=None):
        out = O.dit_stack_f32(latent, t, weights, blocks, ctx, heads, eps, img_ctx=img_ctx, rows=rows)
        return out if rows is None else np.roll(out, 1, axis=0)   # rows returned out of order
    _fails(P.check_stack_f32, ungated_ffn)
    _fails(P.check_stack_f32, last_block_all_rows)


def _mutated(fn, old, new):
    """A copy of oracle function ``fn`` with one source line changed."""
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(fn))
    assert old in src, old
    ns = dict(vars(O))
    exec(src.replace(old, new, 1), ns)
    return ns[fn.__name__]


def test_attention_fp8_running_base_mutations_are_caught(monkeypatch):
    import functools
    base = O._running_base_rows
    mutants = [
        functools.partial(base, warp=1),                  # each row decides alone
        functools.partial(base, threshold=6.0),           # moves too early
        functools.partial(base, block=128),               # key split over 128-row blocks
        _mutated(base, "o *= alpha", "pass"),                                    # output not rescaled
        _mutated(base, "g0, g1 = np.exp2(b0 - bm), np.exp2(b1 - bm)", "g0, g1 = 1.0, 1.0"),  # halves summed
        _mutated(base, "p = prob(St, cr, np.ceil(m * cr), j * tile)", "p = prob(St, cr, m * cr, j * tile)"),  # unrounded base
    ]
    for mut in mutants:
        monkeypatch.setattr(O, "_running_base_rows", mut)
        _fails(P.check_attention_fp8_running_base, O.attention_fp8)
    monkeypatch.setattr(O, "_running_base_rows", base)
    P.check_attention_fp8_running_base(O.attention_fp8)


def test_head_and_image_mlp_mutations_are_caught():
    def no_norm(x, w, b, eps=1e-6):                     # LayerNorm dropped from the head
        return O.linear(x, w, b)

    def eps_outside_head(x, w, b, eps=1e-6):            # eps added to the deviation, not the variance
        x = np.asarray(x, np.float64)
        ln = (x - x.mean(-1, keepdims=True)) / (np.sqrt(x.var(-1, keepdims=True)) + eps)
        return O.linear(ln, w, b)
    _fails(P.check_head, no_norm)
    _fails(P.check_head, eps_outside_head)

    def relu_mlp(feat, w1, b1, w2, b2, w3, b3):         # ReLU for GELU-tanh
        h = np.maximum(O.linear(feat, w1, b1), 0)
        return O.linear(np.maximum(O.linear(h, w2, b2), 0), w3, b3)

    def gelu_on_output(feat, w1, b1, w2, b2, w3, b3):   # activation after the last layer too
        return O.gelu_tanh(O.image_context_mlp(feat, w1, b1, w2, b2, w3, b3))

    def one_gelu(feat, w1, b1, w2, b2, w3, b3):         # the second activation dropped
        return O.linear(O.linear(O.gelu_tanh(O.linear(feat, w1, b1)), w2, b2), w3, b3)
    for mut in (relu_mlp, gelu_on_output, one_gelu):
        _fails(P.check_image_context_mlp, mut)


def test_flow_matching_mutations_are_caught():
    def swapped_ends(x1, x0, u):                         # x_t = t x0 + (1 - t) x1
        return O.flow_matching_input(x0, x1, u)

    def flipped_target(x1, x0):                          # v = x0 - x1
        return O.flow_matching_target(x0, x1)

    def half_step(x1, x0, u):                            # t used as t / 2
        return O.flow_matching_input(x1, x0, u / 2)
    _fails(P.check_flow_matching, swapped_ends, O.flow_matching_target)
    _fails(P.check_flow_matching, O.flow_matching_input, flipped_target)
    _fails(P.check_flow_matching, half_step, O.flow_matching_target)


def test_i2v_input_mutations_are_caught():
    def cond_first(noise, cond, mask):                   # condition latent before the noise
        return O.i2v_input(cond, noise, mask)

    def mask_before_cond(noise, cond, mask):             # mask channels before the condition
        return np.concatenate([np.asarray(noise, np.float64), np.asarray(mask, np.float64),
                               np.asarray(cond, np.float64)], axis=0)
    _fails(P.check_i2v_input, cond_first)
    _fails(P.check_i2v_input, mask_before_cond)


def test_stack_mutations_are_caught():
    def reversed_blocks(latent, t, weights, blocks, ctx, heads, **kw):   # blocks applied last to first
        return O.dit_stack(latent, t, weights, list(blocks)[::-1], ctx, heads, **kw)

    def first_block_twice(latent, t, weights, blocks, ctx, heads, **kw):  # one block's weights for all
        return O.dit_stack(latent, t, weights, [blocks[0]] * len(blocks), ctx, heads, **kw)

    def time_in_thousandths(latent, t, weights, blocks, ctx, heads, **kw):  # t rescaled to [0, 1]
        return O.dit_stack(latent, t / 1000.0, weights, blocks, ctx, heads, **kw)
    for mut in (reversed_blocks, first_block_twice, time_in_thousandths):
        _fails(P.check_stack, mut)
