"""The multi-GPU path is replicas only: every rank runs the whole step on its own
sample, NCCL carries only the barrier and the max-over-ranks timing. These tests run
that host logic with world_size 2 on the gloo backend (CPU): the slowest replica sets
the time, the whole-job throughput counts every replica's tokens, ranks draw different
samples, and the oracle (reference) arm does its work on rank 0 only."""
import importlib.util
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        local_ms = 10.0 + 5.0 * rank                     # rank 1 is the slower replica
        ms = b.max_over_ranks(local_ms, world, "cpu")
        value = b.replica_throughput(world, 32760, ms)
        from wan_inputs import WORKLOADS, make_inputs
        w = WORKLOADS["tiny_f32_block"]
        noise = make_inputs(w, seed=rank, block_input=False)["noise"]
        gathered = [None] * world
        dist.all_gather_object(gathered, noise.sum().item())
        dist.barrier()
        q.put((rank, ms, value, gathered))
    finally:
        dist.destroy_process_group()


def test_replicas_max_over_ranks_and_throughput_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, gathered in out:
        assert ms == 15.0                                  # the max over ranks, on every rank
        assert value == pytest.approx(2 * 32760 / 0.015)   # both replicas' tokens / slowest time
        assert gathered[0] != gathered[1]                  # each replica draws its own sample


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    b = _bench()
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 0, 2
    from wan_inputs import WORKLOADS
    assert b.run_reference(A, WORKLOADS["wan13b_480p_block"]) == 0
    assert capsys.readouterr().out == ""                   # no work, no line on other ranks


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert b.replica_throughput(1, 1000, 2.0) == pytest.approx(500000.0)
