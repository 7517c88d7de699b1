"""The multi-rank bench logic on CPU: two gloo ranks, no GPU.

The path shards by rows with no data-path collective.  The only cross-rank
steps are the max over ranks of the timed region and the whole-job value, plus
rank 0 alone running the reference arm.  These run here with world size 2.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        import numpy as np

        import oracle
        from workloads import synth
        # each rank times a different (fake) region; all must agree on the max
        mine = [10.0 + 5.0 * rank, 1.0 + rank]
        got = bench.max_over_ranks(mine, dist)
        # each rank quantises its own row shard with the oracle; gathering the shards
        # must give the single-process result (the path needs no exchange)
        w = synth.make_config(1, rows=64, cols=256)
        xb = synth.bf16_bits(w.x)
        rb = synth.bf16_bits(w.rhat)
        lo, hi = rank * 32, (rank + 1) * 32
        part = oracle.smooth_rotate_quantize(xb[lo:hi], rb)
        codes = torch.from_numpy(part["codes"].astype(np.int64))
        gathered = [torch.zeros_like(codes) for _ in range(world)]
        dist.all_gather(gathered, codes)
        out[rank] = (got, torch.cat(gathered).numpy().tolist())
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_sharding():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()   # no fork of this (threaded) process
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == [15.0, 2.0]
    import numpy as np

    import oracle
    from workloads import synth
    w = synth.make_config(1, rows=64, cols=256)
    full = oracle.smooth_rotate_quantize(synth.bf16_bits(w.x), synth.bf16_bits(w.rhat))
    assert np.array_equal(np.array(out[0][1]), full["codes"].astype(np.int64))


def test_weak_scaling_value():
    import bench
    # 2 ranks x 297.27 MB each in 0.05 ms -> 11890.9 GB/s whole-job
    v = bench.weak_scaling_value(2, bench.algorithmic_bytes(8192, 14336), 0.05)
    assert v == pytest.approx(2 * 8192 * 14336 * 2.53125 / 0.05e-3 / 1e9)
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
