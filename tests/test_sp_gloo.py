"""The Ulysses decomposition that the sequence-parallel kernels implement, run as two
gloo ranks on the CPU with the oracle for each rank's arithmetic: row shards, q|k|v
head slabs sent with one all-to-all, attention over all tokens for the rank's heads,
outputs returned to their owners with a second all-to-all, then the gated output
projection. The gathered result equals the unsharded self-attention branch."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    from oracle import wan_oracle as O
    from video_diffusion_transformer_wan_b200.sequence_parallel import UlyssesPlan
    from wan_inputs import WORKLOADS, make_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = WORKLOADS["tiny_f32_block"]
    inp = make_inputs(w, seed=5, n_blocks=1)
    blk = inp["blocks"][0]
    x, e = inp["x"][0].astype(np.float64), inp["e"][0]
    L, D, H = x.shape[0], w.dim, w.heads
    plan = UlyssesPlan(world, L, H, D)
    mod = O.block_modulation(e, blk["mod_bias"])
    rows = list(plan.rows(rank))
    h = O.modulate(O.layer_norm(x[rows]), mod[0], mod[1])              # row-local
    qkv = O.linear(h, blk["w_qkv"], blk["b_qkv"])                      # [L/P, 3D]
    send = np.concatenate([qkv[:, plan.qkv_columns(s)] for s in range(world)], axis=0)
    recv = torch.empty(world * plan.rows_local, 3 * plan.rank_cols, dtype=torch.float64)
    dist.all_to_all_single(recv, torch.from_numpy(np.ascontiguousarray(send)))
    mine = recv.numpy()                                                # [L, 3D/P], rows in rank order
    c = plan.rank_cols
    o_heads = O.attention(mine[:, :c], mine[:, c:2 * c], mine[:, 2 * c:], plan.heads_local)
    send_o = np.concatenate([o_heads[list(plan.rows(s))] for s in range(world)], axis=0)
    recv_o = torch.empty(world * plan.rows_local, c, dtype=torch.float64)
    dist.all_to_all_single(recv_o, torch.from_numpy(np.ascontiguousarray(send_o)))
    o_local = np.concatenate(np.split(recv_o.numpy(), world, axis=0), axis=1)   # [L/P, D], source-rank slabs
    y = x[rows] + mod[2] * O.linear(o_local, blk["w_o"], blk["b_o"])
    parts = [torch.empty(plan.rows_local, D, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(parts, torch.from_numpy(y))
    if rank == 0:
        full = torch.cat(parts).numpy()
        hm = O.modulate(O.layer_norm(x), mod[0], mod[1])
        ref = x + mod[2] * O.self_attention_branch(hm, blk, H)
        np.save(out_path, np.stack([full, ref]))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_ulysses_decomposition_gloo(tmp_path, world):
    import torch.multiprocessing as mp
    out = str(tmp_path / "sp.npy")
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    full, ref = np.load(out)
    np.testing.assert_allclose(full, ref, rtol=1e-12, atol=1e-12)


def test_plan_index_maps():
    from video_diffusion_transformer_wan_b200.sequence_parallel import UlyssesPlan
    p = UlyssesPlan(4, 32760, 12, 1536)
    assert p.rows_local == 8190 and p.heads_local == 3 and p.rank_cols == 384
    assert list(p.rows(3))[-1] == 32759 and p.owner(8190) == 1 and p.owner(32759) == 3
    cols = p.qkv_columns(1)
    assert cols[0] == 384 and cols[384] == 1536 + 384 and cols[-1] == 2 * 1536 + 767
    assert sorted(c for s in range(4) for c in p.qkv_columns(s)) == list(range(3 * 1536))
    for bad in [(5, 32760, 12, 1536), (7, 32760, 12, 1536), (9, 72, 72, 9216), (2, 33, 12, 1536), (0, 8, 8, 8)]:
        with pytest.raises(ValueError):
            UlyssesPlan(*bad)
