"""The multi-rank paths of bench.py on CPU: two gloo ranks, no GPU.

Every rank runs its own batch of the workload (the problems are independent,
so there is no collective on the data path); the job's time is the slowest
rank's, taken with all_reduce(MAX); the job's throughput is the work of all
ranks over that time.  Here the oracle stands in for the kernel as each rank's
work, so the test also checks that a rank's result depends on its own inputs
only (a shard computed alone equals the same shard computed in the job).
With --shard heads one workload is split instead: each rank takes a contiguous
range of its batch x kv-head groups (with their query heads), and the ranks'
parts put together must equal the whole computed at once.
"""
import json
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank: int, world: int, port: int, out_dir: str):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import synth
    from synth.workloads import WORKLOADS

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    w = WORKLOADS["tiny_w128_s4"]
    seed = bench.rank_seed(w, rank)
    q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=seed)
    O, LSE = oracle.attention(q, k, v, oracle.Pattern(**w.pattern_args()), w.scale)
    my_ms = 10.0 + 5.0 * rank  # a per-rank "time", different on purpose
    job_ms = bench.max_over_ranks(my_ms, dist, "cpu")
    value = bench.job_tflops(world, 1e9, 3, job_ms)
    gathered = [None] * world
    dist.all_gather_object(gathered, {"rank": rank, "seed": seed, "q0": int(q.ravel()[0])})
    np.save(os.path.join(out_dir, f"O_{rank}.npy"), O)
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"seed": seed, "job_ms": job_ms, "value": value, "gathered": gathered}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(world)]
    # distinct batches per rank
    assert r[0]["seed"] != r[1]["seed"]
    assert not np.array_equal(np.load(tmp_path / "O_0.npy"), np.load(tmp_path / "O_1.npy"))
    assert [g["rank"] for g in r[0]["gathered"]] == [0, 1]
    # the job time is the slowest rank's, seen identically by every rank
    assert r[0]["job_ms"] == r[1]["job_ms"] == 15.0
    # whole-job throughput: all ranks' work over the slowest time
    assert math.isclose(r[0]["value"], 2 * 1e9 * 3 / 15e-3 / 1e12)
    # each shard alone equals the shard in the job
    import bench
    import oracle
    import synth
    from synth.workloads import WORKLOADS
    w = WORKLOADS["tiny_w128_s4"]
    for rank in range(world):
        q, k, v = synth.qkv(w.B, w.Hq, w.Hkv, w.N, w.D, seed=bench.rank_seed(w, rank))
        O, _ = oracle.attention(q, k, v, oracle.Pattern(**w.pattern_args()), w.scale)
        assert np.array_equal(O, np.load(tmp_path / f"O_{rank}.npy"))


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    from synth.workloads import WORKLOADS
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"steps": 3, "warmup": 3, "gpus": 2})()
    assert bench.run_reference(args, WORKLOADS["tiny_w128_s4"]) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_helpers_without_process_group():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert math.isclose(bench.job_tflops(1, 2e12, 10, 1000.0), 20.0)


@pytest.mark.parametrize("n_heads,world", [(16, 2), (16, 3), (8, 8), (5, 2), (1, 1), (64, 7)])
def test_head_shards_partition_the_heads(n_heads, world):
    import bench
    ranges = [bench.shard_heads(n_heads, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == n_heads
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 < a1
    sizes = [h1 - h0 for h0, h1 in ranges]
    assert max(sizes) - min(sizes) <= 1


def shard_rank_main(rank: int, world: int, port: int, out_dir: str):
    """One workload split across the ranks by kv heads (bench --shard heads):
    each rank runs its range of the batch x kv-head groups, as a batch of one,
    with the oracle standing in for the kernel."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    B, Hq, Hkv, N, D = 2, 6, 3, 300, 32
    h0, h1 = bench.shard_heads(B * Hkv, world, rank)
    q, k, v = bench.shard_inputs(*synth.qkv(B, Hq, Hkv, N, D, seed=0), B, Hq, Hkv, h0, h1)
    O, LSE = oracle.attention(q, k, v, oracle.Pattern(window=60, sinks=4), 1 / math.sqrt(D))
    np.save(os.path.join(out_dir, f"shard_O_{rank}.npy"), O)
    np.save(os.path.join(out_dir, f"shard_L_{rank}.npy"), LSE)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_split_one_workload(tmp_path):
    """The ranks' shards put together equal the whole workload computed at once."""
    world = 2
    mp.spawn(shard_rank_main, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    import oracle
    import synth
    B, Hq, Hkv, N, D = 2, 6, 3, 300, 32
    q, k, v = synth.qkv(B, Hq, Hkv, N, D, seed=0)
    O, LSE = oracle.attention(q, k, v, oracle.Pattern(window=60, sinks=4), 1 / math.sqrt(D))
    parts_O = [np.load(tmp_path / f"shard_O_{r}.npy") for r in range(world)]
    parts_L = [np.load(tmp_path / f"shard_L_{r}.npy") for r in range(world)]
    # flattened batch x query-head order: kv head h's query heads are h * g .. h * g + g - 1
    got_O = np.concatenate([x[0] for x in parts_O], axis=0).reshape(O.shape)
    got_L = np.concatenate([x[0] for x in parts_L], axis=0).reshape(LSE.shape)
    assert np.array_equal(got_O, O) and np.array_equal(got_L, LSE)
    assert sum(x.shape[1] for x in parts_O) == B * Hq
