"""Parity of the single kernels (through the C ABI) with the CPU oracle: LayerNorm +
modulation, the GEMM and its epilogues, attention (tails, strided layouts, sharp and
flat softmax), patchify, the timestep MLP, I2V input fusion and flow matching."""
import math

import numpy as np
import pytest

from oracle import wan_oracle as O
from wan_inputs import round_bf16
from gpu_util import BF16_TOL, F32_TOL, dev, host, rel_err, rng

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wan():
    import video_diffusion_transformer_wan_b200 as w
    return w


def _cfg(wan, dtype, D=256, heads=2, ffn=512, **kw):
    return wan.make_config(D, heads, ffn, dtype=dtype, **kw)


def _act(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def _rb(a, dtype):
    return round_bf16(a) if dtype == "bf16" else np.asarray(a, np.float32)


# ------------------------------------------------------------------------------ K-a
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D,B,L", [(128, 1, 32), (1536, 2, 37), (5120, 1, 130), (320, 2, 5), (1536, 1, 1)])
def test_layernorm_modulation(wan, dtype, D, B, L):
    r = rng(D + L)
    cfg = _cfg(wan, dtype, D=D, heads=D // 64)   # layernorm does not use heads
    x = (r.standard_normal((B, L, D)) * 3 + 0.5).astype(np.float32)
    e = (r.standard_normal((B, 6, D)) * 0.3).astype(np.float32)
    mb = (r.standard_normal((6, D)) * 0.1).astype(np.float32)
    xd, ed, mbd = dev(x, torch.float32), dev(e, torch.float32), dev(mb, torch.float32)
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    for chunk in (-1, 0, 1):
        h = torch.empty(B, L, D, dtype=_act(dtype), device="cuda")
        wan.adaln_modulate(cfg, xd, ed, mbd if chunk != 1 else None, chunk, h)
        torch.cuda.synchronize()
        ref = np.empty((B, L, D))
        for b in range(B):
            ln = O.layer_norm(x[b], 1e-6)
            if chunk < 0:
                ref[b] = ln
            else:
                m = O.block_modulation(e[b], mb if chunk != 1 else np.zeros_like(mb))
                ref[b] = O.modulate(ln, m[3 * chunk], m[3 * chunk + 1])
        err = rel_err(host(h), ref)
        assert err <= tol, (chunk, err)
        if dtype == "bf16":
            assert err <= 8e-3   # one bf16 rounding of the output


# ------------------------------------------------------------------------------ K-c
GEMM_SHAPES = [(300, 256, 1536), (129, 384, 192), (77, 64, 64), (50, 1536, 144), (1000, 4608, 128),
               (513, 3072, 1536), (128, 8960 // 4, 256),
               # CTA-pair tiles (M >= 1024, N >= 256, K >= 256): a ragged last pair tile in
               # rows (the odd CTA's half beyond M) and in columns
               (1100, 768, 320), (2200, 1160, 512)]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("epi", ["store", "gelu", "residual", "f32", "residual_nogate"])
def test_linear_epilogues(wan, dtype, M, N, K, epi):
    if dtype == "f32" and M * N * K > 2e8:
        pytest.skip("fp32 SIMT GEMM only serves the small fp32 workload")
    r = rng(M + N + K)
    cfg = _cfg(wan, dtype)
    A = _rb(r.standard_normal((M, K)), dtype)
    W = _rb(r.standard_normal((N, K)) * 0.05, dtype)
    bias = _rb(r.standard_normal(N) * 0.1, dtype)
    Ad, Wd, bd = dev(A, _act(dtype)), dev(W, _act(dtype)), dev(bias, _act(dtype))
    lin = O.linear(A, W, bias)
    rows_per_batch = max(1, M // 2)
    nb = (M + rows_per_batch - 1) // rows_per_batch
    if epi in ("store", "gelu"):
        out = torch.empty(M, N, dtype=_act(dtype), device="cuda")
        wan.linear_fwd(cfg, Ad, Wd, bd, out, wan.EPI_STORE if epi == "store" else wan.EPI_GELU)
        ref = lin if epi == "store" else O.gelu_tanh(lin)
        got = host(out)
    elif epi == "f32":
        out = torch.empty(M, N, dtype=torch.float32, device="cuda")
        wan.linear_fwd(cfg, Ad, Wd, bd, out, wan.EPI_F32)
        ref, got = lin, None
    else:
        x0 = r.standard_normal((M, N)).astype(np.float32)
        out = dev(x0, torch.float32)
        if epi == "residual":
            gate = (r.standard_normal((nb, 3 * N)) * 0.5).astype(np.float32)
            gb = (r.standard_normal(N) * 0.1).astype(np.float32)
            gd, gbd = dev(gate, torch.float32), dev(gb, torch.float32)
            # gate rows live at column offset N of a [nb, 3N] table (batch stride 3N)
            wan.linear_fwd(cfg, Ad, Wd, bd, out, wan.EPI_RESIDUAL, gate=gd[:, N:].data_ptr(), gate_bias=gbd,
                           gate_batch_stride=3 * N, rows_per_batch=rows_per_batch)
            g = gate[np.arange(M) // rows_per_batch, N:2 * N] + gb
            ref = x0 + g * lin
            delta_ref = g * lin
        else:
            wan.linear_fwd(cfg, Ad, Wd, bd, out, wan.EPI_RESIDUAL, rows_per_batch=rows_per_batch)
            ref = x0 + lin
            delta_ref = lin
        torch.cuda.synchronize()
        got = host(out)
        tol = BF16_TOL if dtype == "bf16" else F32_TOL
        assert rel_err(got - x0, delta_ref) <= tol / 4
        return
    torch.cuda.synchronize()
    got = host(out) if got is None else got
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    err = rel_err(got, ref)
    assert err <= tol / (1 if epi in ("store", "gelu") else 4), err


def test_linear_repeatable_bitwise(wan):
    r = rng(5)
    cfg = _cfg(wan, "bf16")
    A, W = dev(round_bf16(r.standard_normal((700, 512))), torch.bfloat16), \
        dev(round_bf16(r.standard_normal((1024, 512)) * 0.05), torch.bfloat16)
    o1 = torch.empty(700, 1024, dtype=torch.float32, device="cuda")
    o2 = torch.empty_like(o1)
    wan.linear_fwd(cfg, A, W, None, o1, wan.EPI_F32)
    wan.linear_fwd(cfg, A, W, None, o2, wan.EPI_F32)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


# ------------------------------------------------------------------------------ K-b
def _attn_case(r, B, Lq, Lk, H, d, sigma):
    q = r.standard_normal((B, Lq, H * d)) * sigma
    k = r.standard_normal((B, Lk, H * d)) * sigma
    v = r.standard_normal((B, Lk, H * d))
    return q, k, v


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,Lq,Lk,H", [(1, 200, 300, 2), (2, 130, 512, 1), (1, 128, 257, 2), (1, 64, 16, 2),
                                       (1, 5, 1, 1), (1, 384, 384, 1), (2, 1, 700, 2), (1, 1000, 129, 1)])
@pytest.mark.parametrize("logit_std", [1.0, 4.0])
def test_attention(wan, dtype, B, Lq, Lk, H, logit_std):
    d = 128 if dtype == "bf16" else 64
    r = rng(Lq * 7 + Lk + H)
    sigma = math.sqrt(logit_std)   # q.k / sqrt(d) then has standard deviation logit_std
    q, k, v = (_rb(a, dtype) for a in _attn_case(r, B, Lq, Lk, H, d, sigma))
    cfg = _cfg(wan, dtype, D=H * d, heads=H)
    o = torch.empty(B, Lq, H * d, dtype=_act(dtype), device="cuda")
    wan.attention_fwd(cfg, dev(q, _act(dtype)), dev(k, _act(dtype)), dev(v, _act(dtype)), o, H, d)
    torch.cuda.synchronize()
    got = host(o)
    tol = BF16_TOL if dtype == "bf16" else F32_TOL
    for b in range(B):
        ref = O.attention(q[b], k[b], v[b], H)
        err = rel_err(got[b], ref)
        assert err <= tol, (b, err)


@pytest.mark.parametrize("B,Lq,Lk,H", [(1, 200, 2100, 2), (2, 130, 2048, 1), (1, 1000, 2000, 1), (2, 1, 4000, 2),
                                       (1, 600, 2500, 3), (1, 300, 1900, 1)])
def test_attention_key_split(wan, B, Lq, Lk, H):
    """With a workspace, units of a last wave that fills at most half of the SMs (here
    every unit) are split over the key tiles (when there are 16 or more) and merged:
    against the oracle, and close to the unsplit call; 1900 keys (15 tiles) stay
    whole."""
    d = 128
    r = rng(Lq * 5 + Lk + H)
    q, k, v = (_rb(a, "bf16") for a in _attn_case(r, B, Lq, Lk, H, d, 2.0))
    cfg = _cfg(wan, "bf16", D=H * d, heads=H)
    qd, kd, vd = dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16)
    o = torch.empty(B, Lq, H * d, dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o)
    ws = torch.empty(max(16, wan.attention_workspace_bytes(cfg, B, Lq)), dtype=torch.uint8, device="cuda")
    wan.attention_fwd(cfg, qd, kd, vd, o, H, d, ws=ws)
    wan.attention_fwd(cfg, qd, kd, vd, o2, H, d)
    torch.cuda.synchronize()
    got = host(o)
    for b in range(B):
        assert rel_err(got[b], O.attention(q[b], k[b], v[b], H)) <= BF16_TOL
    assert rel_err(got, host(o2)) <= 1e-2


def test_attention_planted_peak_and_strided_layout(wan):
    """Self-attention layout (q|k|v packed in one [B, L, 3D] buffer) writing into the
    right half of a [B, L, 2D] buffer; selected query rows get one key equal to 8 q."""
    r = rng(11)
    B, L, H, d = 1, 333, 2, 128
    D = H * d
    qkv = r.standard_normal((B, L, 3 * D))
    rows = [0, 17, 200, 332]
    for i, j in zip(rows, [5, 300, 17, 330]):
        qkv[0, j, D:2 * D] = 8 * qkv[0, i, :D] / math.sqrt(d) * 2
    qkv = round_bf16(qkv)
    cfg = _cfg(wan, "bf16", D=D, heads=H)
    qd = dev(qkv, torch.bfloat16)
    o = torch.zeros(B, L, 2 * D, dtype=torch.bfloat16, device="cuda")
    wan.attention_fwd(cfg, qd, qd, qd, o, H, d, q_col0=0, k_col0=D, v_col0=2 * D, o_col0=D)
    torch.cuda.synchronize()
    got = host(o)
    ref = O.attention(qkv[0, :, :D], qkv[0, :, D:2 * D], qkv[0, :, 2 * D:], H)
    assert rel_err(got[0, :, D:], ref) <= BF16_TOL
    assert np.all(got[0, :, :D] == 0)          # left half untouched
    assert rel_err(got[0, rows, D:], ref[rows]) <= BF16_TOL


def test_attention_running_max_jumps(wan):
    """Rows whose score maximum jumps up in later key tiles, by less and by more than the
    kernel's lazy-rescale threshold (2^8 in exp2 units, 62.7 in raw logits at d = 128),
    so the running base moves (O and the sum rescaled) once or several times per row."""
    r = rng(13)
    B, Lq, H, d = 1, 256, 1, 128
    Lk = 4 * 128 + 50
    q = r.standard_normal((B, Lq, d))
    k = r.standard_normal((B, Lk, d))
    v = r.standard_normal((B, Lk, d))
    plan = {3: [(150, 60.0)], 40: [(130, 80.0), (300, 200.0)], 130: [(260, 70.0), (400, 150.0), (555, 300.0)],
            255: [(520, 90.0), (521, 90.0)]}
    for i, keys in plan.items():
        qi = q[0, i]
        for j, logit in keys:
            k[0, j] = logit * qi * math.sqrt(d) / qi.dot(qi)
    q, k, v = (round_bf16(a) for a in (q, k, v))
    cfg = _cfg(wan, "bf16", D=d, heads=H)
    o = torch.empty(B, Lq, d, dtype=torch.bfloat16, device="cuda")
    wan.attention_fwd(cfg, dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), o, H, d)
    torch.cuda.synchronize()
    got = host(o)
    ref = O.attention(q[0], k[0], v[0], H)
    assert rel_err(got[0], ref) <= BF16_TOL
    rows = sorted(plan)
    assert rel_err(got[0, rows], ref[rows]) <= BF16_TOL
    # row 255's two equal planted keys dominate: its output is their mean value
    np.testing.assert_allclose(got[0, 255], 0.5 * (v[0, 520] + v[0, 521]), atol=2e-2)


def test_attention_long_sequence_sampled_rows(wan):
    r = rng(12)
    B, L, H, d = 1, 4100, 1, 128
    q, k, v = (round_bf16(a) for a in _attn_case(r, B, L, L, H, d, 1.0))
    cfg = _cfg(wan, "bf16", D=128, heads=1)
    o = torch.empty(B, L, d, dtype=torch.bfloat16, device="cuda")
    wan.attention_fwd(cfg, dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), o, H, d)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 2049, 4095, 4096, 4097, 4099])
    ref = O.attention(q[0, rows], k[0], v[0], H)
    assert rel_err(host(o)[0, rows], ref) <= BF16_TOL


# ------------------------------------------------------------------------------ small kernels
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("C", [16, 36])
def test_patchify(wan, dtype, C):
    r = rng(C)
    B, F, H, W, D = 2, 3, 6, 10, 256
    lat = _rb(r.standard_normal((B, C, F, H, W)), dtype)
    wp = _rb(r.standard_normal((D, C, 1, 2, 2)) * 0.05, dtype)
    bp = _rb(r.standard_normal(D) * 0.05, dtype)
    cfg = _cfg(wan, dtype, D=D, in_ch=C)
    L = F * (H // 2) * (W // 2)
    x = torch.empty(B, L, D, dtype=torch.float32, device="cuda")
    ws = torch.empty(B * L * C * 4 * 4, dtype=torch.uint8, device="cuda")
    wan.patchify(cfg, dev(lat, _act(dtype)), dev(wp.reshape(D, -1), _act(dtype)), dev(bp, _act(dtype)), x, ws)
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.patchify(lat[b], wp, bp)
        assert rel_err(host(x)[b], ref) <= (1e-5 if dtype == "f32" else 1e-3)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("D", [128, 1536, 5120])
def test_time_mlp(wan, dtype, D):
    r = rng(D)
    B = 3
    t = np.array([0.0, 431.25, 999.9], np.float32)
    w1, b1 = _rb(r.standard_normal((D, 256)) * 0.02, dtype), _rb(r.standard_normal(D) * 0.02, dtype)
    w2, b2 = _rb(r.standard_normal((6 * D, D)) * 0.02, dtype), _rb(r.standard_normal(6 * D) * 0.02, dtype)
    cfg = _cfg(wan, dtype, D=D, heads=D // 64 if dtype == "f32" else D // 128)
    ts = [dev(a, _act(dtype)) for a in (w1, b1, w2, b2)]
    tw = wan.TimeWeights(*(x.data_ptr() for x in ts))
    e = torch.empty(B, 6, D, dtype=torch.float32, device="cuda")
    wan.time_mlp(cfg, dev(t, torch.float32), tw, e)
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.time_mlp(float(t[b]), w1, b1, w2, b2)
        assert rel_err(host(e)[b], ref) <= F32_TOL


def test_i2v_input_exact(wan):
    r = rng(3)
    B, F, H, W = 2, 3, 4, 6
    noise, cond = round_bf16(r.standard_normal((B, 16, F, H, W))), round_bf16(r.standard_normal((B, 16, F, H, W)))
    keep = np.zeros((B, 1 + 4 * (F - 1)), np.uint8)
    keep[0, 0] = 1
    keep[1, 8] = 1
    cfg = _cfg(wan, "bf16")
    out = torch.empty(B, 36, F, H, W, dtype=torch.bfloat16, device="cuda")
    wan.i2v_input(cfg, dev(noise, torch.bfloat16), dev(cond, torch.bfloat16),
                  torch.from_numpy(keep).cuda(), out)
    torch.cuda.synchronize()
    got = host(out)
    for b in range(B):
        ref = O.i2v_input(noise[b], cond[b], O.i2v_mask(keep[b], F, H, W))
        assert np.array_equal(got[b], ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_flow_matching(wan, dtype):
    r = rng(4)
    B, n = 2, 16 * 3 * 4 * 6
    x1, x0 = _rb(r.standard_normal((B, n)), dtype), _rb(r.standard_normal((B, n)), dtype)
    u = np.array([0.25, 0.8], np.float32)
    cfg = _cfg(wan, dtype)
    xt = torch.empty(B, n, dtype=_act(dtype), device="cuda")
    t = torch.empty(B, dtype=torch.float32, device="cuda")
    x1d, x0d = dev(x1, _act(dtype)), dev(x0, _act(dtype))
    wan.flow_matching_input(cfg, x1d, x0d, dev(u, torch.float32), xt, t)
    v = r.standard_normal((B, n)).astype(np.float32)
    loss = torch.empty(B, dtype=torch.float32, device="cuda")
    wan.flow_matching_loss(cfg, dev(v, torch.float32), x1d, x0d, loss)
    torch.cuda.synchronize()
    for b in range(B):
        ref = O.flow_matching_input(x1[b], x0[b], float(u[b]))
        assert rel_err(host(xt)[b], ref) <= (1e-6 if dtype == "f32" else 4e-3)
        ref_loss = np.mean((v[b] - O.flow_matching_target(x1[b], x0[b])) ** 2)
        assert abs(float(loss[b]) - ref_loss) / ref_loss < 1e-5
    assert np.allclose(t.cpu().numpy(), 1000 * u)


def test_bounded_wait_reports_timeout_and_context_survives(wan):
    """A wait on a barrier that nothing arrives at gives up after its limit; the host
    reads WAN_ERR_TIMEOUT once, the flag clears, and the next kernel runs normally."""
    assert wan.device_status() == 0
    wan.wait_timeout_check()
    assert wan.device_status() == -7
    assert wan.device_status() == 0
    cfg = _cfg(wan, "bf16", D=128, heads=1)
    q = dev(rng(31).standard_normal((1, 130, 128)), torch.bfloat16)
    o = torch.empty(1, 130, 128, dtype=torch.bfloat16, device="cuda")
    wan.attention_fwd(cfg, q, q, q, o, 1, 128)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    ref = O.attention(host(q)[0], host(q)[0], host(q)[0], 1)
    assert rel_err(host(o)[0], ref) <= BF16_TOL
