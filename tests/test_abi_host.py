"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports every
function include/wan.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wan.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(wan_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def wan():
    from video_diffusion_transformer_wan_b200 import build
    build.build()
    import video_diffusion_transformer_wan_b200 as w
    return w


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ["wan_patchify", "wan_adaln_modulate", "wan_self_attn_fwd", "wan_cross_attn_fwd", "wan_ffn_fwd",
                     "wan_dit_block_fwd", "wan_dit_stack_fwd", "wan_workspace_bytes", "wan_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(wan):
    lib = ctypes.CDLL(wan.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(wan):
    for code in range(0, -9, -1):
        assert wan.status_string(code) and wan.status_string(code) != "unknown status"
    assert wan.status_string(-100) == "unknown status"


def _cfg(wan, **kw):
    d = dict(dim=1536, heads=12, ffn=8960, dtype="bf16")
    d.update(kw)
    return wan.make_config(**d)


def test_workspace_bytes_layout(wan):
    cfg = _cfg(wan)
    B, L, Lc = 1, 32760, 512
    n = wan.workspace_bytes(cfg, B, L, Lc)
    D, F = 1536, 8960
    # h + max(5LD + 2LcD, LF) act elements + fp32 x + fp32 e, each region 256-aligned,
    # + partial outputs for at most 74 key-split attention units (2 x 2 x 128 rows x 520 B)
    split = min(B * 12 * ((L + 255) // 256), 74) * 2 * 2 * 128 * 520
    lower = 2 * (B * L * D + max(5 * L * D + 2 * Lc * D, L * F)) + 4 * (B * L * D + 6 * D) + split
    assert lower <= n <= lower + 5 * 256
    assert wan.workspace_bytes(cfg, 2, L, Lc) > n
    assert wan.workspace_bytes(_cfg(wan, heads=7), 1, 10, 10) == 0       # D != heads * head_dim


def test_validation_rejects_before_launch(wan):
    """Bad arguments return negative statuses without touching the GPU (pointers are
    never dereferenced on the host, and no launch happens on a validation error)."""
    L = wan.lib
    launches = wan.launch_count()
    cfg = _cfg(wan)
    fake = 1 << 20                      # 16-byte aligned fake device address
    bw = wan.BlockWeights(*([fake] * 17))
    # NULL x
    st = L.wan_dit_block_fwd(ctypes.byref(cfg), None, fake, fake, 512, None, 0, ctypes.byref(bw), 1, 32, fake,
                             1 << 40, None)
    assert st == -1
    # misaligned x
    st = L.wan_dit_block_fwd(ctypes.byref(cfg), fake + 4, fake, fake, 512, None, 0, ctypes.byref(bw), 1, 32, fake,
                             1 << 40, None)
    assert st == -4
    # workspace too small
    st = L.wan_dit_block_fwd(ctypes.byref(cfg), fake, fake, fake, 512, None, 0, ctypes.byref(bw), 1, 32, fake, 16, None)
    assert st == -5
    # empty text context
    st = L.wan_dit_block_fwd(ctypes.byref(cfg), fake, fake, fake, 0, None, 0, ctypes.byref(bw), 1, 32, fake,
                             1 << 40, None)
    assert st == -2
    # unknown dtype
    bad = _cfg(wan)
    bad.dtype = 7
    assert L.wan_dit_block_fwd(ctypes.byref(bad), fake, fake, fake, 512, None, 0, ctypes.byref(bw), 1, 32, fake,
                               1 << 40, None) == -3
    # bf16 with head_dim 64 is not implemented by the tensor-core attention
    c64 = _cfg(wan, dim=128, heads=2, ffn=256)
    assert L.wan_dit_block_fwd(ctypes.byref(c64), fake, fake, fake, 16, None, 0, ctypes.byref(bw), 1, 32, fake,
                               1 << 40, None) == -8
    # odd latent width for patchify
    assert L.wan_patchify(ctypes.byref(cfg), fake, 1, 2, 8, 7, fake, fake, fake, fake, 1 << 30, None) == -2
    # I2V block without the image K/V weight
    bw2 = wan.BlockWeights(*([fake] * 17))
    bw2.w_ckv_img = None
    assert L.wan_dit_block_fwd(ctypes.byref(cfg), fake, fake, fake, 512, fake, 257, ctypes.byref(bw2), 1, 32, fake,
                               1 << 40, None) == -1
    # attention: heads must match the config
    assert L.wan_attention_fwd(ctypes.byref(cfg), fake, 4608, 0, fake, 4608, 1536, fake, 4608, 3072, fake, 1536, 0,
                               1, 11, 32, 32, 128, None, 0, None) == -2
    assert wan.attention_workspace_bytes(cfg, 1, 32760) == 74 * 2 * 2 * 128 * 520   # 1536 units: capped at 74
    assert wan.attention_workspace_bytes(cfg, 1, 256) == 12 * 2 * 2 * 128 * 520     # 12 units
    # linear: N must be a multiple of 8
    assert L.wan_linear_fwd(ctypes.byref(cfg), fake, fake, None, fake, 32, 12, 64, 0, None, None, 0, 1, None) == -2
    assert wan.launch_count() == launches


def test_sampler_validation_and_workspace(wan):
    """The sampling call checks its arguments before any launch; its workspace covers
    the 2B-sample stack pass plus the per-block K|V caches."""
    L = wan.lib
    launches = wan.launch_count()
    cfg = _cfg(wan)
    fake = 1 << 20
    bws = (wan.BlockWeights * 2)(*[wan.BlockWeights(*([fake] * 17)) for _ in range(2)])
    sw = wan.StackWeights(fake, fake, wan.TimeWeights(fake, fake, fake, fake), fake, fake)
    B, F, H, W, Lc = 1, 21, 60, 104, 512
    need = wan.sample_workspace_bytes(cfg, 2, B, F, H, W, Lc)
    Lt = F * (H // 2) * (W // 2)
    assert need > wan.workspace_bytes(cfg, 2 * B, Lt, Lc) + 2 * 2 * (2 * B * Lc * 2 * 1536)
    assert wan.sample_workspace_bytes(_cfg(wan, heads=7), 2, B, F, H, W, Lc) == 0

    def call(n_steps=4, g=5.0, c=cfg, ctx_u=fake, ws=1 << 40, b=B, h=H, cache=None):
        return L.wan_sample_euler_cfg(ctypes.byref(c), 2, fake, b, F, h, W, n_steps, g, ctypes.byref(sw), bws, fake,
                                      ctx_u, Lc, None, 0, None if cache is None else ctypes.byref(cache), None, fake,
                                      fake, ws, None)
    assert call(n_steps=0) == -2
    assert call(g=float("nan")) == -2
    assert call(g=float("inf")) == -2
    assert call(ctx_u=None) == -1
    assert call(ws=need - 1) == -5
    assert call(h=59) == -2
    c2 = _cfg(wan, in_ch=16, out_ch=20)
    assert call(c=c2) == -2
    assert call(b=0) == 0
    assert call(cache=wan.DiffusionCache(1, 0, 2, 2)) == -2          # interval 0
    assert call(cache=wan.DiffusionCache(-1, 2, 2, 2)) == -2         # negative start
    kept = wan.sample_workspace_bytes(cfg, 2, B, F, H, W, Lc, cache=wan.DiffusionCache(1, 2, 3, 2))
    assert kept - need >= 2 * 2 * B * Lt * 1536 * 2 + B * 16 * F * H * W * 4      # attention outputs + residual
    assert call(cache=wan.DiffusionCache(1, 2, 3, 2), ws=kept - 1) == -5
    assert wan.launch_count() == launches


def test_trace_read_without_events(wan):
    assert wan.trace_read(wan.KIND_ATTN) == (0.0, 0)


def test_binding_refuses_strided_views(wan):
    """The C calls take dense row-major arrays; a strided view is refused before the
    call instead of being read with the wrong layout."""
    import torch
    t = torch.zeros(4, 6)
    assert wan._p(t) == t.data_ptr()
    with pytest.raises(ValueError):
        wan._p(t.t())
    with pytest.raises(ValueError):
        wan._p(t[:, 1:3])
    assert wan._p_strided(t[:, 2]) == t[:, 2].data_ptr()


def test_empty_inputs_launch_nothing(wan):
    """Zero samples or zero tokens are valid and do nothing: status 0, no launch (which is
    why this runs without a GPU)."""
    L = wan.lib
    cfg = _cfg(wan)
    fake = 1 << 20
    bw = wan.BlockWeights(*([fake] * 17))
    n = wan.launch_count()
    for B, T in [(0, 32), (1, 0), (0, 0)]:
        assert L.wan_dit_block_fwd(ctypes.byref(cfg), fake, fake, fake, 512, None, 0, ctypes.byref(bw), B, T, fake,
                                   1 << 40, None) == 0
        assert L.wan_self_attn_fwd(ctypes.byref(cfg), fake, ctypes.byref(bw), fake, fake, B, T, fake, 1 << 40,
                                   None) == 0
        assert L.wan_ffn_fwd(ctypes.byref(cfg), fake, ctypes.byref(bw), fake, fake, B, T, fake, 1 << 40, None) == 0
    assert L.wan_attention_fwd(ctypes.byref(cfg), fake, 4608, 0, fake, 4608, 1536, fake, 4608, 3072, fake, 1536, 0,
                               0, 12, 32, 32, 128, None, 0, None) == 0
    assert L.wan_linear_fwd(ctypes.byref(cfg), fake, fake, None, fake, 0, 64, 64, 0, None, None, 0, 1, None) == 0
    assert wan.launch_count() == n


def test_attention_fp8_validation_and_workspace(wan):
    """8-bit attention: workspace = q codes + q scales + k codes + v^T codes (keys padded
    to a multiple of 64) + k/v scales + the key-split scratch, each 256-aligned; bad
    arguments are refused before any launch."""
    L = wan.lib
    cfg = _cfg(wan)
    B, Lq, Lk, H, D = 1, 32760, 32760, 12, 1536
    n = wan.attention_fp8_workspace_bytes(cfg, B, Lq, Lk)
    S = (Lk + 63) // 64 * 64
    split = min(B * H * ((Lq + 255) // 256), 74) * 2 * 2 * 128 * 520
    lower = B * Lq * D + 4 * B * Lq * H + B * Lk * D + B * D * S + 8 * B * H + split
    assert lower <= n <= lower + 6 * 256
    assert wan.attention_fp8_workspace_bytes(_cfg(wan, dtype="f32"), B, Lq, Lk) == 0
    assert wan.attention_fp8_workspace_bytes(cfg, B, Lq, 0) == 0
    fake = 1 << 20
    n0 = wan.launch_count()

    def fwd(c=cfg, ws_bytes=1 << 40, heads=H, hd=128, lk=Lk, q_col0=0, ws=fake):
        return L.wan_attention_fp8_fwd(ctypes.byref(c), fake, 3 * D, q_col0, fake, 3 * D, D, fake, 3 * D, 2 * D, fake,
                                       D, 0, B, heads, Lq, lk, hd, ws, ws_bytes, None)
    assert fwd(ws_bytes=n - 1) == -5                     # workspace too small
    assert fwd(ws=None) == -1                            # workspace required
    assert fwd(c=_cfg(wan, dtype="f32")) == -8           # bf16 only
    assert fwd(heads=8) == -2 and fwd(hd=64) == -2       # heads / head_dim differ from the config
    assert fwd(lk=0) == -2                               # no keys
    assert fwd(q_col0=3 * D) == -2                       # head columns past the row
    q = L.wan_attention_fp8_quantize
    args = (ctypes.byref(cfg), fake, 3 * D, 0, fake, 3 * D, D, fake, 3 * D, 2 * D, B, H, Lq, Lk, 128, fake, fake,
            fake, fake)
    assert q(*args, S - 1, fake, None) == -2             # v^T row stride not a multiple of 64
    assert q(*args, S - 64, fake, None) == -2            # shorter than the keys
    assert q(*args[:-1], fake + 8, S, fake, None) == -4  # v^T codes not 16-byte aligned
    assert wan.launch_count() == n0


def test_missing_library_fails_loudly(tmp_path):
    """With the CUDA library absent, the first call raises: there is no CPU fallback."""
    import subprocess
    import sys
    code = ("import video_diffusion_transformer_wan_b200 as w\n"
            "try:\n"
            "    w.status_string(0)\n"
            "except ImportError as e:\n"
            "    print('refused:', e)\n"
            "    raise SystemExit(3)\n")
    env = dict(os.environ, WAN_B200_LIB=str(tmp_path / "absent.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=120)
    assert r.returncode == 3 and "refused:" in r.stdout


def test_fp8_workspace_holds_the_bf16_workspace_codes_and_attention_operands(wan):
    """FP8 block workspace = the bf16 block's + E4M3 codes of the widest activation
    (F or D per row) and of the context + their row scales + the 8-bit self-attention's
    operands (its own key-split scratch excluded: the block's is reused), each region
    256-aligned; the FP8 sampler's is larger than the bf16 sampler's by that much."""
    cfg = _cfg(wan)
    B, L, Lc, H, D, F = 1, 32760, 512, 12, 1536, 8960
    base = wan.workspace_bytes(cfg, B, L, Lc)
    S = (L + 63) // 64 * 64
    attn = B * L * D + 4 * B * L * H + B * L * D + B * D * S + 8 * B * H
    extra = B * L * max(F, D) + B * Lc * D + 4 * B * L + 4 * B * Lc + attn
    n = wan.fp8_workspace_bytes(cfg, B, L, Lc)
    assert base + extra <= n <= base + extra + 10 * 256
    assert wan.fp8_workspace_bytes(_cfg(wan, heads=7), B, 10, 10) == 0


def test_both_patchify_calls_accept_and_reject_the_same_arguments(wan):
    """wan_patchify and wan_patchify_noalloc run the same argument checks before any
    launch: a config that one refuses, the other refuses with the same status."""
    L = wan.lib
    f = L.wan_patchify_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(wan.Config), ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    launches = wan.launch_count()
    fake = 1 << 20
    bad = []
    c = _cfg(wan, heads=7)                      # dim != heads * head_dim
    bad.append((c, -2))
    c = _cfg(wan)
    c.eps = 0.0                                 # eps must be positive
    bad.append((c, -2))
    c = _cfg(wan, out_ch=15)                    # odd output channels
    bad.append((c, -2))
    c = _cfg(wan, freq_dim=12)                  # frequency dim not a multiple of 8
    bad.append((c, -2))
    c = _cfg(wan, ffn=100)                      # FFN width not a multiple of 64
    bad.append((c, -2))
    c = _cfg(wan)
    c.dtype = 5                                 # unknown dtype
    bad.append((c, -3))
    for cfg, code in bad:
        a = L.wan_patchify(ctypes.byref(cfg), fake, 1, 2, 8, 8, fake, fake, fake, fake, 1 << 30, None)
        b = f(ctypes.byref(cfg), fake, 1, 2, 8, 8, fake, fake, fake, None)
        assert a == b == code, (a, b, code)
    cfg = _cfg(wan)
    # null and misaligned pointers, odd width: the same status from both
    for args in [(0, fake, fake), (fake + 8, fake, fake), (fake, fake + 4, fake), (fake, fake, fake + 2)]:
        lat, wp, out = args
        a = L.wan_patchify(ctypes.byref(cfg), lat or None, 1, 2, 8, 8, wp, fake, out, fake, 1 << 30, None)
        b = f(ctypes.byref(cfg), lat or None, 1, 2, 8, 8, wp, fake, out, None)
        assert a == b and a < 0, (args, a, b)
    assert L.wan_patchify(ctypes.byref(cfg), fake, 1, 2, 8, 7, fake, fake, fake, fake, 1 << 30, None) == \
        f(ctypes.byref(cfg), fake, 1, 2, 8, 7, fake, fake, fake, None) == -2
    # token counts whose product with the batch passes 2^31 are refused as a shape, not
    # by a wrapped workspace size
    assert L.wan_patchify(ctypes.byref(cfg), fake, 1 << 12, 1 << 10, 1 << 6, 1 << 6, fake, fake, fake, fake,
                          1 << 62, None) == -2
    assert wan.launch_count() == launches
