"""Host-side logic of bench.py's multi-GPU mode (independent replicas, weak
scaling), exercised with two gloo ranks on the CPU."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(values[rank])
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, [1.5, 3.25], out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == 3.25 and out[1] == 3.25


def test_max_over_ranks_alone_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(2.5) == 2.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload = "tiny_256x512x512_r16"
        steps = 1
        warmup = 3

    out, rank = bench.run_reference(Args())
    assert out is None and rank == 1


@pytest.mark.parametrize("ws", [1, 2])
def test_reference_arm_line_on_rank_zero(monkeypatch, ws, capsys):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", str(ws))

    class Args:
        workload = "tiny_256x512x512_r16"
        steps = 1
        warmup = 3

    out, rank = bench.run_reference(Args())
    assert rank == 0 and out["impl"] == "reference" and out["n_gpus"] == ws
    assert out["value"] > 0 and out["cpu_baseline"]["kind"] == "oracle"
    assert out["e2e"]["h2d_bytes_per_step"] == 0
