"""Multi-rank logic of bench.py on CPU: two gloo ranks (world size 2).

bench.py runs one process per GPU under torchrun, one call's heads split
round-robin over the ranks; the rank-level pieces it relies on are the
barrier, the max and sum of per-rank values over all ranks, the ms per call,
the rank-0-only reference line and the head-sharded call itself.  They are checked
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
        per_call = bench.call_ms(10.0 * (rank + 1), 5, world)
        total = bench.sum_over_ranks(1.0 + rank, world)
        bench.barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": mx, "per_call": per_call, "sum": total}, f)
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
        assert r["per_call"] == pytest.approx(20.0 / 5)  # 5 calls, each spread over both ranks
        assert r["sum"] == 3.0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    bench.barrier(1)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.call_ms(30.0, 3, 1) == pytest.approx(10.0)
    assert bench.sum_over_ranks(2.5, 1) == 2.5


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


# --------------------------------------------------------------------------- head sharding
def _host_scope_heads(q, k, v, params, grid):
    """Per-head SCOPE call on the host (the oracle), standing in for the
    library on gloo ranks that have no GPU: [B, H', N, D] float64 output."""
    import numpy as np

    import oracle

    p = params
    B, Hl, N, D = q.shape
    out = torch.empty((B, Hl, N, D), dtype=torch.float64)
    for b in range(B):
        for h in range(Hl):
            pl = oracle.scope_plan_head(q[b, h].double().numpy(), k[b, h].double().numpy(), p)
            o = oracle.scope_attn_head(pl["qr"], pl["kr"], v[b, h].double().numpy(), pl["q_labels"], pl["lists"])
            out[b, h] = torch.from_numpy(np.ascontiguousarray(o))
    return out


def _shard_worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import oracle
    from cluster_guided_sparse_b200 import shard, synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.WORKLOADS["tiny"].with_(H=3)  # 3 heads over 2 ranks: {0, 2} and {1}
        q, k, v = synth.make_inputs(w)
        p = oracle.Params.of(w)
        local = shard.sharded_attention(q, k, v, p, None, gather=False, run=_host_scope_heads)
        full = shard.sharded_attention(q, k, v, p, None, run=_host_scope_heads)
        # a rank that holds only its own heads (pass the total head count)
        mine = shard.heads_of(w.H, rank, world)
        own = shard.sharded_attention(q[:, mine], k[:, mine], v[:, mine], p, None, H=w.H,
                                      run=_host_scope_heads)
        torch.save({"local": local, "full": full, "own": own, "heads": mine},
                   os.path.join(out_dir, f"shard{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_head_sharded_call_equals_single_rank(tmp_path):
    sys.path.insert(0, ROOT)
    import oracle
    from cluster_guided_sparse_b200 import shard, synth

    world = 2
    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    w = synth.WORKLOADS["tiny"].with_(H=3)
    q, k, v = synth.make_inputs(w)
    ref = shard.sharded_attention(q, k, v, oracle.Params.of(w), None, run=_host_scope_heads)  # no group: 1 rank
    seen = []
    for r in range(world):
        res = torch.load(tmp_path / f"shard{r}.pt")
        assert res["heads"] == shard.heads_of(3, r, world) == [h for h in range(3) if h % world == r]
        assert torch.equal(res["local"], ref[:, res["heads"]])  # each rank computed exactly its heads
        assert torch.equal(res["full"], ref)  # the all-gather reassembles every head in place
        assert torch.equal(res["own"], ref)
        seen += res["heads"]
    assert sorted(seen) == [0, 1, 2]


def test_head_partition_rules():
    sys.path.insert(0, ROOT)
    from cluster_guided_sparse_b200 import shard

    for H in (1, 3, 24, 40):
        for world in (1, 2, 3, 8):
            parts = [shard.heads_of(H, r, world) for r in range(world)]
            assert sorted(h for p in parts for h in p) == list(range(H))
            assert max(map(len, parts)) - min(map(len, parts)) <= 1
    x = torch.arange(2 * 5 * 3 * 4, dtype=torch.float32).view(2, 5, 3, 4)
    assert torch.equal(shard.local_heads(x, 1, 2), x[:, [1, 3]])
    with pytest.raises(ValueError):
        shard.heads_of(4, 2, 2)
