"""Ulysses sequence parallelism through the C ABI, all ranks emulated on one GPU (each
phase for every rank, then the next phase; local buffers stand in for the peers'):
the sharded self-attention branch equals the unsharded call bitwise and the oracle
within the bf16 bar, with every element of the exchange buffers written."""
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


@pytest.mark.parametrize("P,frames,height,width", [(2, 3, 20, 28), (4, 3, 20, 28), (2, 2, 16, 16), (1, 2, 16, 16)])
def test_sharded_self_attention(wan, P, frames, height, width):
    from video_diffusion_transformer_wan_b200.sequence_parallel import UlyssesPlan, emulate_self_attn
    w = small_bf16(frames=frames, height=height, width=width, dim=512, heads=4, ffn=1024, batch=2)
    r = Run(wan, w, zero_wx=False)
    B, L, D = w.batch, w.tokens, w.dim
    plan = UlyssesPlan(P, L, w.heads, D)
    bw, mb, blk = r.model.block_tables[0], r.model.blocks[0]["mod_bias"], r.inp["blocks"][0]
    h = torch.empty(B, L, D, dtype=r.act, device="cuda")
    wan.adaln_modulate(r.cfg, r.x, r.e, mb, 0, h)
    # unsharded reference through the single-kernel calls (attention without a workspace,
    # so every work unit runs whole, as in the sharded attention)
    blk_dev = r.model.blocks[0]
    qkv_full = torch.empty(B, L, 3 * D, dtype=r.act, device="cuda")
    wan.linear_fwd(r.cfg, h, blk_dev["w_qkv"], blk_dev["b_qkv"], qkv_full, wan.EPI_STORE)
    o_full = torch.empty(B, L, D, dtype=r.act, device="cuda")
    wan.attention_fwd(r.cfg, qkv_full, qkv_full, qkv_full, o_full, w.heads, D // w.heads, 0, D, 2 * D, 0)
    x_ref = r.x.clone()
    wan.linear_fwd(r.cfg, o_full, blk_dev["w_o"], blk_dev["b_o"], x_ref, wan.EPI_RESIDUAL, gate=r.e[:, 2],
                   gate_bias=mb[2], gate_batch_stride=6 * D, rows_per_batch=L)
    # sharded
    rows = [list(plan.rows(k)) for k in range(P)]
    h_shards = [h[:, rows[k]].contiguous() for k in range(P)]
    x_shards = [r.x[:, rows[k]].contiguous() for k in range(P)]
    nan = float("nan")
    qkv_bufs = [torch.full(plan.qkv_shape(B), nan, dtype=r.act, device="cuda") for _ in range(P)]
    o_bufs = [torch.full(plan.shard_shape(B), nan, dtype=r.act, device="cuda") for _ in range(P)]
    emulate_self_attn(wan, r.cfg, plan, h_shards, bw, r.e, x_shards, qkv_bufs, o_bufs)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    for k in range(P):
        assert torch.equal(qkv_bufs[k], qkv_full[:, :, plan.qkv_columns(k)])
        assert not torch.isnan(o_bufs[k]).any()
    x_sp = torch.cat(x_shards, dim=1)
    assert torch.equal(x_sp, x_ref)
    got = host(x_sp)
    for b in range(B):
        mod = O.block_modulation(r.inp["e"][b], blk["mod_bias"])
        hm = O.modulate(O.layer_norm(r.inp["x"][b]), mod[0], mod[1])
        assert rel_err(got[b] - r.inp["x"][b], mod[2] * O.self_attention_branch(hm, blk, w.heads)) <= BF16_TOL


def test_sp_validation(wan):
    """Bad group sizes and shapes are refused before any launch."""
    import ctypes
    w = small_bf16(frames=2, height=16, width=16, dim=512, heads=4, ffn=1024)
    r = Run(wan, w)
    L = wan.lib
    bufs = (ctypes.c_void_p * 8)(*([r.ws.data_ptr()] * 8))
    bw = ctypes.byref(r.model.block_tables[0])
    n = wan.launch_count()
    assert L.wan_sp_qkv_fwd(ctypes.byref(r.cfg), 3, 0, r.ws.data_ptr(), 1, 128, bw, bufs, None) == -2   # 4 % 3
    assert L.wan_sp_qkv_fwd(ctypes.byref(r.cfg), 2, 2, r.ws.data_ptr(), 1, 128, bw, bufs, None) == -2   # rank
    assert L.wan_sp_qkv_fwd(ctypes.byref(r.cfg), 2, 0, r.ws.data_ptr(), 1, 127, bw, bufs, None) == -2   # L % P
    assert L.wan_sp_attn_fwd(ctypes.byref(r.cfg), 9, 0, r.ws.data_ptr(), 1, 144, bufs, None) == -2      # P > 8
    assert L.wan_sp_attn_fwd(ctypes.byref(r.cfg), 2, 0, r.ws.data_ptr(), 1, 128, None, None) == -1
    assert wan.launch_count() == n
