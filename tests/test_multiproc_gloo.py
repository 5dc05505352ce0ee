"""The N > 1 host path of bench.py on CPU: two gloo ranks exercise the
max-over-ranks step time and the whole-job (weak-scaling) throughput, and the
reference arm's rank gating. No GPU and no GPU collective is involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        # each rank measured a different step time; the job's is the max
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
        value = bench.weak_scaling_value(w, 100.0, ms * 1e-3)
        out[rank] = (ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_whole_job_value():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, value in res.values():
        assert ms == 15.0                       # the slowest rank
        assert value == pytest.approx(2 * 100.0 / 0.015)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.weak_scaling_value(1, 10.0, 2.0) == 5.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, gpus = 1, 0, 2
    assert bench.run_reference(A) == 0
    assert capsys.readouterr().out == ""
