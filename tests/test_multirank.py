"""Multi-rank logic of bench.py on CPU: two gloo ranks (world size 2).

bench.py runs one process per GPU under torchrun; the rank-level pieces it
relies on are the barrier, the max of a per-rank time over all ranks, the
whole-job ms-per-call and the rank-0-only reference line.  They are checked
here with a gloo process group on 127.0.0.1, no GPU involved.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # rank r "measured" 10 * (r + 1) ms for its steps
        mx = bench.max_over_ranks(10.0 * (rank + 1), world)
        per_call = bench.job_ms_per_call(10.0 * (rank + 1), 5, world)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "per_call": per_call}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_agree_on_max_and_job_rate(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 20.0  # the slowest rank's time, on every rank
        assert r["per_call"] == pytest.approx(20.0 / (5 * 2))  # 5 calls per rank, 2 ranks


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    bench.barrier(1)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_ms_per_call(30.0, 3, 1) == pytest.approx(10.0)


def test_reference_arm_prints_nothing_off_rank0(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    args = argparse.Namespace(workload="hunyuan720p", warmup=3, steps=5, gpus=2)
    bench.run_reference(args, world=2, rank=1)
    assert capsys.readouterr().out == ""


def test_tile_flops_counts_padded_tiles():
    sys.path.insert(0, ROOT)
    import bench

    sizes = torch.tensor([0, 1, 128, 129, 256, 257])
    n = torch.tensor([5, 128, 129, 1, 256, 300])
    # Q tiles x key tiles per cluster: 0, 1x1, 1x2, 2x1, 2x2, 3x3
    assert bench.tile_flops(sizes, n, 128) == 4.0 * 128 * 128 * 128 * 18


def test_reference_arm_line_has_the_contract_keys(capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    args = argparse.Namespace(workload="tiny", warmup=1, steps=1, gpus=1)
    bench.run_reference(args, world=1, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["higher_is_better"] is False and line["value"] > 0
    for key in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "scaling", "dtype", "data", "config"):
        assert key in line, key
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
