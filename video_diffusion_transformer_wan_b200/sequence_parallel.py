"""Ulysses sequence parallelism for the DiT block's self-attention (the intra-machine
layer of the context parallelism described on the Wan 2.1 pages: 163.com article on
Wan2.1, "核心创新三"; Wan 2.1 page, "Infra", 2D CP = outer Ring Attention x inner Ulysses).

P ranks split every sample's L tokens into P contiguous shards. Everything in a block
except self-attention is row-local and runs on the shard with the ordinary calls. Self-
attention runs in three phases of the C ABI, each of which stores its result straight
into the buffers of the ranks that consume it:

  1. ``wan_sp_qkv_fwd``  h_shard W_qkv^T + b -> every rank's head slab, at this shard's rows
  2. ``wan_sp_attn_fwd`` attention over all L tokens for this rank's H/P heads -> every
                         row's owner, at this rank's head columns
  3. ``wan_sp_out_fwd``  o_shard W_o^T + b, gated residual into this shard of x

``UlyssesPlan`` is the index arithmetic the kernels implement (also used by the CPU
tests). ``emulate_self_attn`` runs all P ranks on one GPU, one phase at a time, with
local buffers standing in for the peers'. ``UlyssesGroup`` is the one-process-per-GPU
form: its buffers live in symmetric memory so that every rank's kernels can store into
its peers', and a barrier between phases orders them across ranks.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

MAX_RANKS = 8


@dataclass(frozen=True)
class UlyssesPlan:
    world: int
    L: int          # tokens per sample (all ranks)
    heads: int
    dim: int

    def __post_init__(self):
        if not 1 <= self.world <= MAX_RANKS:
            raise ValueError(f"sequence-parallel size {self.world} is outside 1..{MAX_RANKS}")
        if self.heads % self.world or self.L % self.world:
            raise ValueError(f"heads ({self.heads}) and tokens ({self.L}) must divide by {self.world}")

    @property
    def rows_local(self) -> int:
        return self.L // self.world

    @property
    def heads_local(self) -> int:
        return self.heads // self.world

    @property
    def rank_cols(self) -> int:
        """Columns of one of q, k, v that a rank attends over (its heads)."""
        return self.dim // self.world

    def rows(self, rank: int) -> range:
        return range(rank * self.rows_local, (rank + 1) * self.rows_local)

    def heads_of(self, rank: int) -> range:
        return range(rank * self.heads_local, (rank + 1) * self.heads_local)

    def qkv_columns(self, rank: int) -> List[int]:
        """Columns of the [L, 3D] projection that rank `rank` receives, in the order of
        its [L, 3D/P] buffer: its q slab, then its k slab, then its v slab."""
        c0 = rank * self.rank_cols
        return [part * self.dim + c0 + c for part in range(3) for c in range(self.rank_cols)]

    def owner(self, row: int) -> int:
        """Rank that owns token `row` of a sample."""
        return row // self.rows_local

    def qkv_shape(self, B: int):
        return (B, self.L, 3 * self.rank_cols)

    def shard_shape(self, B: int):
        return (B, self.rows_local, self.dim)


def emulate_self_attn(wan, cfg, plan: UlyssesPlan, h_shards: Sequence, bw, e, x_shards: Sequence,
                      qkv_bufs: Sequence, o_bufs: Sequence, stream=None) -> None:
    """All P ranks on one GPU: phase 1 for every rank, then phase 2, then phase 3. Stream
    order stands in for the barrier between phases."""
    P = plan.world
    for r in range(P):
        wan.sp_qkv_fwd(cfg, P, r, h_shards[r], plan.L, bw, qkv_bufs, stream)
    for r in range(P):
        wan.sp_attn_fwd(cfg, P, r, qkv_bufs[r], plan.L, o_bufs, stream)
    for r in range(P):
        wan.sp_out_fwd(cfg, P, o_bufs[r], bw, e, x_shards[r], plan.L, stream)


class UlyssesGroup:
    """One process per GPU over a torch.distributed group (NCCL). The qkv and o buffers
    are allocated in symmetric memory; the pointer tables hold the peers' addresses."""

    def __init__(self, plan: UlyssesPlan, B: int, group=None):
        import torch
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        self.plan, self.B = plan, B
        self.group = group if group is not None else dist.group.WORLD
        self.rank = dist.get_rank(self.group)
        if dist.get_world_size(self.group) != plan.world:
            raise ValueError("group size differs from the plan")
        act = torch.bfloat16
        self.qkv = symm_mem.empty(*plan.qkv_shape(B), dtype=act, device="cuda")
        self.o = symm_mem.empty(*plan.shard_shape(B), dtype=act, device="cuda")
        self._hq = symm_mem.rendezvous(self.qkv, self.group)
        self._ho = symm_mem.rendezvous(self.o, self.group)
        self.qkv_peers = [self._hq.get_buffer(s, plan.qkv_shape(B), act) for s in range(plan.world)]
        self.o_peers = [self._ho.get_buffer(s, plan.shard_shape(B), act) for s in range(plan.world)]

    def _barrier(self):
        self._hq.barrier(channel=0)

    def self_attn(self, wan, cfg, h_shard, bw, e, x_shard, stream=None) -> None:
        P, r, L = self.plan.world, self.rank, self.plan.L
        wan.sp_qkv_fwd(cfg, P, r, h_shard, L, bw, self.qkv_peers, stream)
        self._barrier()
        wan.sp_attn_fwd(cfg, P, r, self.qkv, L, self.o_peers, stream)
        self._barrier()
        wan.sp_out_fwd(cfg, P, self.o, bw, e, x_shard, L, stream)
