"""Multi-process host logic of bench.py on CPU: two gloo ranks.

The benchmark runs one process per GPU under torchrun; each rank times its
own replica and the job's time is the maximum over ranks. Here two CPU
processes (gloo) exercise the same initialisation, barrier, max-over-ranks
and whole-job arithmetic, and the reference arm's rule that only rank 0
times the oracle.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, elapsed, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_init(world)
    bench.barrier(w)
    m = bench.max_over_ranks(elapsed[rank], w)
    value, ms = bench.whole_job_value(m, steps=3, n_loops=4, world=w)
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, w, m, value, ms))


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port, elapsed = _free_port(), [12.5, 30.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, elapsed, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, m, value, ms) in enumerate(got):
        assert (rank, world) == (r, 2)
        assert m == 30.0                          # both ranks see the maximum
        # 2 ranks x 3 steps x 4 loop steps done in 30 ms
        assert value == pytest.approx(30.0e3 / 24)
        assert ms == pytest.approx(10.0)


def test_whole_job_value_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    value, ms = bench.whole_job_value(40.0, steps=10, n_loops=4, world=1)
    assert value == pytest.approx(1000.0) and ms == pytest.approx(4.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_encoder_bound_fractions():
    import bench
    b1 = bench.encode_bounds(1000, 16, 1e-3)
    assert b1["bytes"] == 1000 * (16 * 2 + 16 * 4 + 1)
    assert b1["flops"] == 1000 * 2 * 32 * 256
    assert b1["alu_ops"] == 1000 * 256 * 3
    b2 = bench.encode_bounds(1000, 16, 2e-3)
    for k in ("hbm_frac", "tensor_frac", "alu_frac"):
        assert abs(b2[k] * 2 - b1[k]) < 1e-12 * b1[k]


def test_call_percentiles():
    import bench
    assert bench.call_percentiles(list(range(11))) == [1, 5, 9]
    assert bench.call_percentiles([3.0]) == [3.0, 3.0, 3.0]
    assert all(v != v for v in bench.call_percentiles([]))      # NaN
