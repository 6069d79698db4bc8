"""Multi-rank host logic on the CPU (gloo, two ranks).

The decode shards by stream: every rank decompresses its own blocks, so the
only cross-rank steps are the timing barrier, the maximum over ranks of the
elapsed time and the all-ranks bit-exact flag.  These run here under gloo
exactly as bench.py runs them under NCCL on GPUs.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from tests.conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [12.5, 20.0][rank]             # rank 1 is the slow one
        t = bench.max_over_ranks(elapsed, "cpu")
        exact = bench.min_over_ranks(rank == 0, "cpu")
        seed = bench.rank_seed_offset(rank)
        dist.barrier()
        q.put((rank, t, exact, seed))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_flags_under_gloo():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [20.0, 20.0]       # everyone sees the slowest rank
    assert [o[2] for o in out] == [False, False]     # one rank not exact -> not exact
    assert out[0][3] != out[1][3]                    # different blocks per rank


def test_aggregate_counts_all_ranks_over_the_slowest_time():
    a = bench.aggregate([10.0, 20.0], bytes_per_rank_step=1_000_000_000, steps=4)
    assert a["ms"] == 20.0 and a["ms_per_step"] == 5.0
    assert a["gbs"] == pytest.approx(2 * 4 * 1e9 / 20e-3 / 1e9)
    one = bench.aggregate([10.0], 1_000_000_000, 4)
    assert one["gbs"] == pytest.approx(400.0)


def test_helpers_without_process_group():
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.min_over_ranks(True, "cpu") is True


def test_reference_arm_under_torchrun_two_ranks():
    """Rank 0 alone runs the CPU oracle and prints one JSON line; rank 1
    exits without work."""
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3", "--ref-sample", "20000"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 3
    assert d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_parallel_oracle_baseline_reproduces_the_input():
    # the bench's multi-threaded CPU baseline: ranges of thread blocks decoded
    # on host threads through Gaps and block offsets, checked against x
    import numpy as np
    import bench
    from lossless_entropy_coded_dfloat11_b200 import inputs as I
    x = I.edge_case(70001, "zipf", 12).flat_u16()
    dt, s = bench.time_oracle_decode(x, 1, 0)
    assert dt > 0
    for threads in (1, 3):
        dtp, y = bench.time_oracle_decode_parallel(s, x, threads)
        assert dtp > 0 and np.array_equal(y, x)
