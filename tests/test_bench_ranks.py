"""Host logic of bench.py for more than one rank, on CPU with two gloo ranks: the
device time is the max over ranks, throughput counts every rank's tokens, and the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 30.0][rank]               # rank 1 is the slow one
        m = bench.max_over_ranks(my_ms, world, "cpu")
        out[rank] = (m, bench.throughput(world, 4, 10, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        m, v = out[r]
        assert m == 30.0                          # both ranks see the slowest rank's time
        assert v == pytest.approx(2 * 4 * 10 / 0.030)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(7.0, 1, None) == 7.0
    assert bench.throughput(1, 1, 100, 50.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup = 1, 3

    assert bench.run_reference(Args(), synth.CONFIGS[2]) == 0
    assert capsys.readouterr().out == ""


def test_paths_and_launch_counts():
    import dataclasses
    c2, c3, c4 = synth.CONFIGS[2], synth.CONFIGS[3], synth.CONFIGS[4]
    # one token: the router, gate/up (K in parts), the K-part reduction, down, combine
    assert bench.path_of(c2) == "decode" and bench.decode_kparts(c2)[0] > 1
    assert bench.launches_per_step(c2) == 1 + 3 + 1
    # 5 to 8 tokens: the router, then the whole forward as one kernel
    for T in (5, 6, 8):
        c = dataclasses.replace(c2, T=T)
        assert bench.path_of(c) == "fused" and bench.launches_per_step(c) == 1 + 1
    # 3, 4, 16 and 24 tokens: the separate decode kernels
    for T in (3, 4):
        assert bench.path_of(dataclasses.replace(c2, T=T)) == "decode"
    assert bench.path_of(c3) == "decode"
    c24 = dataclasses.replace(c2, T=24)
    assert bench.path_of(c24) == "decode"
    assert bench.launches_per_step(c24) == 1 + 3 + (1 if bench.decode_kparts(c24)[0] > 1 else 0)
    assert bench.path_of(c4) == "prefill" and bench.launches_per_step(c4) == 3 + 4
