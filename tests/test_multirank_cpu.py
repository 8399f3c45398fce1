"""Host logic of the N > 1 benchmark path, on CPU with the gloo backend and two
ranks: timings are reduced as the max over ranks, whole-job throughput counts
every rank's units (weak scaling, independent replicas, no collective on the
data path), and only rank 0 prints the reference arm's line."""
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


def _worker(rank, world, port, times, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, _ = bench.dist_env()
    dist.init_process_group("gloo", init_method="env://", rank=r, world_size=w,
                            timeout=__import__("datetime").timedelta(seconds=60))
    ms = bench.reduce_max(times[rank], w, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    out_q.put((rank, ms, bench.job_rate(1000, w, ms)))


def test_reduce_max_and_job_rate_gloo_two_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [12.5, 20.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time; the job processed 2 x 1000 units
    for rank, ms, rate in res:
        assert ms == 20.0
        assert rate == pytest.approx(2 * 1000 / 0.020)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1, "cpu") == 3.5
    assert bench.job_rate(200000, 1, 5000.0) == pytest.approx(40000.0)


def test_reference_arm_only_rank0_prints():
    # rank 1 of a 2-rank launch exits 0 without work and without output
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_pattern_of_matches_ratio():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.pattern_of(8, 4) == "FSSSFSSS"
    assert bench.pattern_of(48, 4).count("F") == 12
