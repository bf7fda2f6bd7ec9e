"""The multi-process path of bench.py on the host: two gloo ranks on
127.0.0.1 (no GPU). Every rank must see the slowest rank's time, the job's
rate is the units of all ranks over that time, and the reference arm does no
work on the ranks other than 0."""
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


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow replica
        m = bench.max_over_ranks(ms, ws, torch.device("cpu"))
        rate = bench.replica_rate(ws, 1000.0, 4, m)
        out[rank] = (m, rate, bench.dist_env())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_the_job_rate():
    ws = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(ws, port, out), nprocs=ws, join=True)
        res = dict(out)
    for rank in range(ws):
        m, rate, env = res[rank]
        assert m == 15.0
        assert rate == pytest.approx(ws * 1000.0 * 4 / 0.015)
        assert env == (ws, rank, rank)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.replica_rate(1, 10.0, 2, 1.0) == pytest.approx(20000.0)


def test_reference_arm_is_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 1, "warmup": 3})()
    assert bench.run_reference(args) is None  # returns at once, prints nothing
    assert capsys.readouterr().out == ""
