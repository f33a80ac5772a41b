"""Host logic of the N-GPU bench path on CPU: two gloo ranks on 127.0.0.1.

Every rank runs its own replica of the workload (weak scaling, no data-path
collective); the only cross-rank steps are the barrier and the max over ranks
of the device-timed milliseconds, from which rank 0 reports the whole-job
throughput. The reference arm runs on rank 0 only.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench.barrier(world, cuda=False)
        local_ms = [3.0, 5.0][rank]  # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world, device="cpu")
        v = bench.aggregate_steps_per_s(world, 10, 32, m)
        bench.barrier(world, cuda=False)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    os.environ["PYTHONPATH"] = ROOT + os.pathsep + os.environ.get("PYTHONPATH", "")
    mgr = mp.get_context("spawn").Manager()  # no fork of a multi-threaded process
    out = mgr.dict()
    mp.spawn(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True)
    for rank in (0, 1):
        m, v = out[rank]
        assert m == 5.0                          # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 10 * 32 / 5e-3)  # units of both ranks over that time


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.aggregate_steps_per_s(1, 4, 32, 2.0) == pytest.approx(4 * 32 / 2e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from cached_block_attention_b200 import synth

    class Args:
        steps, warmup, gpus = 1, 0, 2
    bench.run_reference(Args, synth.WORKLOADS["tiny"], rank=1, world=2)
    assert capsys.readouterr().out == ""
