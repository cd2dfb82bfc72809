"""Host logic of the multi-GPU benchmark path, on CPU with two gloo ranks.

The draft step shards by request: every rank runs its own replica and the step
has no collective.  What crosses ranks is only the timing: the timed region's
length is the max over ranks, and the whole-job rate counts every rank's
blocks.  The reference arm runs on rank 0 alone; other ranks exit at once."""
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


def _rank_main(rank, world, port, times, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], "cpu")
        rate = bench.whole_job_rate(world, 1, 100, ms)
        q.put((rank, ms, rate))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run_ranks(times):
    world = len(times)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    out = sorted(q.get(timeout=5) for _ in range(world))
    return out


def test_time_is_max_over_ranks_and_rate_counts_all_ranks():
    out = _run_ranks([40.0, 55.5])
    for rank, ms, rate in out:
        assert ms == 55.5
        assert rate == pytest.approx(2 * 100 / 0.0555)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, "cpu") == 12.5
    assert bench.whole_job_rate(1, 4, 10, 20.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    # a non-zero rank returns at once, without loading the oracle or any input
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=120,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
