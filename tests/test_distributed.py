"""The N > 1 path of bench.py on CPU: world-size-2 process groups over gloo.

bench.py runs one replica of the workload per GPU (no data-path collective);
the only cross-rank steps are the max-over-ranks reduction of the timed
region and the whole-job throughput derived from it.  These tests run those
steps on two gloo ranks, and check that the reference arm does its work on
rank 0 only.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's own step time; the slowest sets the job's time
        own_ms = 1.5 * (rank + 1)
        ms = bench.max_over_ranks(own_ms)
        value = bench.job_throughput(32768, world, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["ms"] == pytest.approx(3.0)                       # the slower rank's time
        assert g["value"] == pytest.approx(32768 * 2 / 3.0e-3)     # all ranks' units / that time


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25) == 2.25
    assert bench.job_throughput(10, 1, 2.0) == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    from lm_causal_depthwise_b200 import workloads as W
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args, W.TINY_F32) == 0
    assert capsys.readouterr().out == ""


def test_shard_heads_covers_every_head_once():
    sys.path.insert(0, ROOT)
    from lm_causal_depthwise_b200.sharding import shard_heads
    for H in (1, 10, 16):
        for world in (1, 2, 3, 4, 8, 12):
            got = [shard_heads(H, world, r) for r in range(world)]
            heads = [h for a, b in got for h in range(a, b)]
            assert heads == list(range(H))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


def _shard_rank_main(rank: int, world: int, port: int, out_dir: str):
    """Each gloo rank slices its heads of one workload and times a fake step;
    the job's throughput counts the tokens once (strong scaling)."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    from lm_causal_depthwise_b200 import workloads as W
    from lm_causal_depthwise_b200.sharding import shard_heads, shard_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = W.Workload("s", B=2, T=40, D=768, io="bf16", seed=3, init_state="random")
        inp = W.generate(w)
        h0, h1 = shard_heads(w.H, world, rank)
        part = shard_inputs(inp, h0, h1)
        ms = bench.max_over_ranks(1.0 + rank)
        value = bench.sharded_throughput(w.tokens, ms)
        np.save(os.path.join(out_dir, f"x{rank}.npy"), part["x"])
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"h": [h0, h1], "ms": ms, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_sharded_job_gloo(tmp_path):
    """Two ranks take heads [0, 2) and [2, 3) of a 3-head workload; their
    slices of x put back together are the whole x, and the job's time is the
    slower rank's."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from lm_causal_depthwise_b200 import workloads as W
    world = 2
    mp.start_processes(_shard_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [g["h"] for g in got] == [[0, 2], [2, 3]]
    for g in got:
        assert g["ms"] == pytest.approx(2.0)
        assert g["value"] == pytest.approx(2 * 40 / 2.0e-3)
    whole = W.generate(W.Workload("s", B=2, T=40, D=768, io="bf16", seed=3, init_state="random"))["x"]
    parts = [np.load(tmp_path / f"x{r}.npy") for r in range(world)]
    np.testing.assert_array_equal(np.concatenate(parts, axis=2), whole)


def test_shard_time_covers_every_token_once():
    sys.path.insert(0, ROOT)
    from lm_causal_depthwise_b200.sharding import shard_time
    for T in (1, 5, 131072, 4097):
        for world in (1, 2, 3, 8):
            got = [shard_time(T, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [t1 - t0 for t0, t1 in got]
            assert max(sizes) - min(sizes) <= 1


def test_conv_halo_takes_the_three_inputs_before_the_chunk():
    """Chunks starting at 0, 1, 2 take (some of) the carried conv state, later
    ones the last three tokens of x before them, oldest first."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from lm_causal_depthwise_b200.sharding import conv_halo
    x = np.arange(2 * 10 * 4, dtype=np.float32).reshape(2, 10, 4)
    cs = -np.arange(2 * 3 * 4, dtype=np.float32).reshape(2, 3, 4) - 1
    np.testing.assert_array_equal(conv_halo(x, cs, 0), cs)
    np.testing.assert_array_equal(conv_halo(x, cs, 1), np.concatenate([cs[:, 1:], x[:, :1]], axis=1))
    np.testing.assert_array_equal(conv_halo(x, cs, 2), np.concatenate([cs[:, 2:], x[:, :2]], axis=1))
    np.testing.assert_array_equal(conv_halo(x, cs, 7), x[:, 4:7])


def _time_rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    from lm_causal_depthwise_b200.sharding import shard_time
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank's chunk end states (stand-ins); the one exchange gathers them in rank order
        t0, t1 = shard_time(1000, world, rank)
        H0 = torch.full((2, 8), float(rank), dtype=torch.float32)
        H1 = H0 + 0.5
        g0 = [torch.empty_like(H0) for _ in range(world)]
        g1 = [torch.empty_like(H1) for _ in range(world)]
        dist.all_gather(g0, H0)
        dist.all_gather(g1, H1)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"t": [t0, t1], "H0": [float(g[0, 0]) for g in g0], "A": [float(a[0, 0] - b[0, 0])
                                                                                  for a, b in zip(g1, g0)]}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_time_sharded_exchange_gloo(tmp_path):
    """Two ranks split 1000 tokens and gather each other's chunk end states in
    rank order (the input of rglru_carry_scan on every rank)."""
    world = 2
    mp.start_processes(_time_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [g["t"] for g in got] == [[0, 500], [500, 1000]]
    for g in got:
        assert g["H0"] == [0.0, 1.0]
        assert g["A"] == [0.5, 0.5]
