"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each with its own
timing; the reported time is the slowest rank's and the rate is whole-job."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist
    r, w, local = bench.dist_init(world, backend="gloo")
    bench.barrier(w)
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w, torch.device("cpu"))
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump([r, w, local, ms], f)
    dist.destroy_process_group()


def test_two_ranks_report_the_slowest_time(tmp_path):
    # results come back through files: no forked manager process in the test runner
    world, port = 2, _free_port()
    mp.spawn(_rank, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    res = {r: json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)}
    for r, (rank, w, local, ms) in res.items():
        assert (rank, w, local) == (r, 2, r)
        assert ms == 15.0


def test_job_throughput_is_whole_job():
    assert bench.job_throughput(4, 32768, 2.0) == pytest.approx(4 * 32768 / 2e-3)


def test_world_size_mismatch_is_refused(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_init(1, backend="gloo")
