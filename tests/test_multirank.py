"""Host logic of the multi-GPU benchmark path, run as world_size-2 gloo ranks
on the CPU: the per-rank time is reduced with a max over ranks, the replica
value scales with the number of ranks, and the reference arm runs on rank 0
only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slower replica
        m = bench.max_over_ranks(ms, dist, "cpu")
        v = bench.replica_value(1e12, m, world)
        dist.barrier()
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_replica_value():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(2 * 1e12 / 15e-3 / 1e12)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from precision_moe_numerics_quantize_b200 import synth

    class A:
        router = "uniform"
        steps = warmup = 1
        gpus = 2
        workload = "small_moe"

    monkeypatch.setenv("RANK", "1")
    bench.run_reference(A(), synth.SHAPES["small_moe"])
    assert capsys.readouterr().out == ""
