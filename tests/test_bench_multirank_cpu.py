"""The benchmark's multi-rank plumbing on CPU: two gloo ranks agree on the slowest rank's time and
on the whole-job (weak-scaling) rate, the way `bench.py --gpus N` aggregates its timings."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 20.0][rank]
        worst = bench.max_over_ranks(my_ms, world, torch.device("cpu"))
        rate = bench.whole_job_rate(8192.0, world, worst)
        bench.barrier(world)
        out[rank] = (worst, rate)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_max_time_and_rate():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:  # no fork of this multi-threaded process
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    worst, rate = res[0]
    assert worst == 20.0
    assert rate == pytest.approx(2 * 8192.0 / 0.020)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(100.0, 1, 1000.0) == pytest.approx(100.0)


def test_captured_traffic_follows_the_kernel_sources(tmp_path):
    """The roofline's DRAM traffic comes from the committed ncu capture only while the kernel's
    sources hash to the value recorded with it; any other hash (or workload) gives None."""
    import json

    import bench

    real = bench.kernel_source_hash("chunk_local_tc")
    assert real and bench.kernel_source_hash("no_such_kernel") is None
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"chunk_local_tc": {"workload": "w", "dram_bytes_per_launch": 123,
                              "source_sha256": real}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    path = str(prof / "traffic.json")
    assert bench.captured_traffic("chunk_local_tc", "w", path) == 123
    assert bench.captured_traffic("chunk_local_tc", "other", path) is None
    assert bench.captured_traffic("chunk_state_tc", "w", path) is None
    rec["chunk_local_tc"]["source_sha256"] = "0" * 64
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.captured_traffic("chunk_local_tc", "w", path) is None
