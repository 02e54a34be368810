"""Data-parallel host logic of bench.py on CPU ranks (gloo, world size 2):
the job's time is the slowest rank's, its work the sum of every rank's, and
each rank draws its own synthetic sample."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        el, fl = bench.reduce_over_ranks(10.0 + 5.0 * rank, 100.0 * (rank + 1), "cpu")
        out[rank] = (el, fl)
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for rank in range(world):
        el, fl = res[rank]
        assert el == 15.0          # max over ranks
        assert fl == 300.0         # sum over ranks


def test_single_process_is_identity():
    assert bench.reduce_over_ranks(3.5, 7.0, "cpu") == (3.5, 7.0)


def test_ranks_draw_distinct_samples():
    w = synth.WORKLOADS[2]
    a = synth.make_qkv(w.wid, bench.rank_sample(0), 2, 4, 4, 1, 64)[0]
    b = synth.make_qkv(w.wid, bench.rank_sample(1), 2, 4, 4, 1, 64)[0]
    assert not (a == b).all()


def test_bench_spawns_ranks_and_splits_heads(tmp_path):
    """bench.py --gpus 2 (not under a launcher) starts its own two ranks through
    torch.distributed.run; with --plan-only they meet over gloo on the host and
    rank 0 reports each rank's heads and the max-time / summed-work reduction."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    for shard, heads in (("heads", [[0, 6], [6, 12]]), ("samples", [[0, 12], [0, 12]])):
        r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                            "--plan-only", "--shard", shard],
                           capture_output=True, text=True, timeout=300, env=env, cwd=root)
        assert r.returncode == 0, r.stderr[-2000:]
        line = [x for x in r.stdout.splitlines() if x.startswith("{")]
        assert len(line) == 1                      # rank 0 alone prints
        rep = json.loads(line[0])
        assert rep["world"] == 2 and rep["shard"] == shard
        assert [p["heads"] for p in rep["plan"]] == heads
        samples = [p["sample"] for p in rep["plan"]]
        assert samples == ([0, 0] if shard == "heads" else [0, 1])
        assert rep["max_ms"] == 11.0 and rep["work"] == 3.0


def test_head_ranges_cover_every_head_once():
    from block_sparse_attention_layer_b200.sharding import head_range, local_shape
    from block_sparse_attention_layer_b200 import LayerShape
    for n_heads in (1, 5, 12, 13):
        for world in (1, 2, 3, 4, 8, 16):
            got = [head_range(r, world, n_heads) for r in range(world)]
            flat = [h for a, b in got for h in range(a, b)]
            assert flat == list(range(n_heads))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
            assert sizes == sorted(sizes, reverse=True)
    sh = LayerShape(24, 36, 64, 12, 128, 2, 4, 6, 8)
    assert local_shape(sh, 1, 5).n_heads == 3 and local_shape(sh, 4, 5).n_heads == 2
    assert local_shape(sh, 12, 16) is None
