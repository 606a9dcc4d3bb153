"""The N > 1 harness of bench.py on CPU: two gloo ranks (world size 2) exercise the rank logic that the GPU run
uses over NCCL -- per-rank seeding of independent batches (weak scaling, no data-path collective), the barrier,
and the step time taken as the max over ranks."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, local_ms, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        worst = bench.max_over_ranks(local_ms[rank], world, "cpu")
        cfg = dict(bench.WORKLOADS["qwen3_8b"], vocab=64, depths=16)
        inp = bench.make_inputs(cfg, bench.rank_seed(rank))
        q.put((rank, worst, float(np.abs(inp["q"]).sum()), int(inp["roots"][0])))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    local_ms = [0.25, 0.75]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, local_ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    # every rank sees the slowest rank's time
    assert [g[1] for g in got] == [0.75, 0.75]
    # each rank draws its own batch
    assert got[0][2] != got[1][2]


def test_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # weak scaling: N ranks each verify batch * budget nodes in the (max-over-ranks) step time
    assert bench.job_nodes_per_sec(batch=2, budget=64, world=4, step_ms=0.5) == pytest.approx(4 * 2 * 64 / 0.5e-3)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
