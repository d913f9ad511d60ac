"""Host-side logic of bench.py, including the multi-rank path on CPU (gloo, 2 ranks).

The decode path has no data exchange: ranks run independent replicas and only
the timing is reduced (max over ranks).  These tests run that reduction and the
throughput arithmetic without a GPU.
"""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [12.5, 30.0]
        mx = bench.reduce_max(times[rank], torch.device("cpu"))
        rate = bench.whole_job_tokens_per_s(world, 512, 10, mx)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": mx, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_weak_scaling_rate(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert res[0] == res[1]
    assert res[0]["max"] == 30.0
    assert res[0]["rate"] == pytest.approx(2 * 512 * 10 / 0.030)


def test_single_process_reduction_is_identity():
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_tokens_per_s(1, 512, 256, 1000.0) == pytest.approx(512 * 256)


def test_algorithmic_bytes_follow_the_pending_fill():
    # one sequence, fill 255: step 0 reads 256 pending rows, then the block empties
    b0 = bench.algorithmic_read_bytes([255], 0, 1)
    b1 = bench.algorithmic_read_bytes([255], 1, 1)
    per_group_fixed = 2 * 4 * 512 + 2 * 4 * 1024
    assert b0 == 4 * ((2048 + 256) * 1024 + per_group_fixed)
    assert b1 == 4 * ((2048 + 1) * 1024 + per_group_fixed)
