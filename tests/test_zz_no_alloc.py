"""wan_patchify_noalloc: patchify for callers that cannot allocate device memory.

Some callers of this library cannot hand it a workspace: code running where the CUDA
allocator must not be called, plug-ins that receive only input and output pointers
from their host framework, or processes whose device-memory budget is fixed at
start-up. wan_patchify_noalloc gives them the patchify step with its scratch in a
fixed array inside the library. This test calls it through the C ABI and compares it
with wan_patchify (caller-provided workspace) on two calls in a row: the second call
has a different, smaller shape, so whatever the first call left in the shared array
must not leak into it. It also checks that a request above the array's size is
refused before any launch.

The file is named to be collected last, so a run that stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20   # WAN_PATCHIFY_NOALLOC_SCRATCH_BYTES in include/wan.h


def _fn(wan):
    f = wan._lib().wan_patchify_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(wan.Config), ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _case(wan, dtype, B, C, F, H, W, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    act = torch.bfloat16 if dtype == "bf16" else torch.float32
    lat = torch.randn(B, C, F, H, W, device="cuda", generator=g).to(act)
    wp = (torch.randn(D, C * 4, device="cuda", generator=g) * 0.05).to(act)
    bp = (torch.randn(D, device="cuda", generator=g) * 0.05).to(act)
    cfg = wan.make_config(D, D // 64, 4 * D, in_ch=C, dtype=dtype)
    return cfg, lat, wp, bp


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_patchify_noalloc_matches_workspace_patchify_on_two_calls(dtype):
    import video_diffusion_transformer_wan_b200 as wan
    from oracle import wan_oracle as O
    from gpu_util import BF16_TOL, F32_TOL, rel_err
    fn = _fn(wan)
    stream = torch.cuda.current_stream().cuda_stream
    # first call: the 480P latent grid (4.2 MB of bf16 patches), then a smaller I2V-width one
    shapes = [(1, 16, 21, 60, 104, 1536), (2, 36, 3, 6, 10, 256)] if dtype == "bf16" else \
        [(1, 16, 4, 16, 16, 256), (2, 36, 2, 6, 10, 128)]
    for i, (B, C, F, H, W, D) in enumerate(shapes):
        cfg, lat, wp, bp = _case(wan, dtype, B, C, F, H, W, D, seed=i)
        L = F * (H // 2) * (W // 2)
        ref = torch.empty(B, L, D, dtype=torch.float32, device="cuda")
        ws = torch.empty(B * L * C * 4 * 4, dtype=torch.uint8, device="cuda")
        wan.patchify(cfg, lat, wp, bp, ref, ws)
        got = torch.full((B, L, D), float("nan"), dtype=torch.float32, device="cuda")
        st = fn(ctypes.byref(cfg), lat.data_ptr(), B, F, H, W, wp.data_ptr(), bp.data_ptr(), got.data_ptr(), stream)
        assert st == 0, wan.status_string(st)
        torch.cuda.synchronize()
        assert wan.device_status() == 0
        # the same gather and the same GEMM kernel as wan_patchify: bit for bit equal, so
        # nothing left in the shared array by the previous call can hide in a tolerance
        assert torch.equal(got, ref), (i, (got - ref).abs().max().item())
        # and the oracle's strided convolution, at the dtype's bar, on the last sample
        b = B - 1
        want = O.patchify(lat[b].float().cpu().numpy(), wp.float().cpu().numpy().reshape(D, C, 1, 2, 2),
                          bp.float().cpu().numpy())
        err = rel_err(got[b].cpu().numpy(), want)
        assert err <= (BF16_TOL if dtype == "bf16" else F32_TOL), (i, err)


def test_patchify_noalloc_rejects_requests_above_its_scratch():
    import video_diffusion_transformer_wan_b200 as wan
    fn = _fn(wan)
    cfg = wan.make_config(1536, 12, 8960, in_ch=36)
    fake = 1 << 20
    # 36 channels x 4 x 2 bytes per token: 2 x 21 x 45 x 80 tokens need 43.5 MB > 16 MiB
    st = fn(ctypes.byref(cfg), fake, 2, 21, 90, 160, fake, fake, fake, None)
    assert st == -2
    assert 2 * 21 * 45 * 80 * 36 * 4 * 2 > SCRATCH_BYTES
