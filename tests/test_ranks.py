"""The N > 1 path of bench.py on CPU: two processes over gloo (127.0.0.1).

bench.py runs one independent replica per GPU (the layer has no cross-token
exchange), so its multi-rank logic is the barrier, the max of the ranks'
timed durations and the whole-job throughput; only rank 0 prints.  The GPU
work itself is not involved."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [12.5, 20.0][rank]                    # rank 1 is the slower one
        dist.barrier()
        m = bench.max_over_ranks(ms, dist, "cpu")
        v = bench.job_tokens_per_s(world, 21, 100, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 20.0                           # every rank sees the slowest duration
        assert v == pytest.approx(2 * 21 * 100 / 0.020)


def test_single_process_passes_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, None, "cpu") == 7.0
    assert bench.job_tokens_per_s(1, 21, 10, 1000.0) == pytest.approx(210.0)


def test_reference_arm_prints_on_rank_zero_only():
    # rank 1 of a 2-rank reference run exits 0 without work or output
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
