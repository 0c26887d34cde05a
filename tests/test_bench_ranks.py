"""bench.py's multi-rank arithmetic, on CPU with the gloo backend.

With N > 1 every rank runs its own batch (the layer has no cross-token
exchange, so ranks are independent replicas); the job's time is the slowest
rank's and the job's throughput counts every rank's tokens.  These tests run
world-size-2 process groups over gloo and check that the timing reduction and
the aggregate follow that rule, and that the reference arm's second rank exits
without work.
"""
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, local_ms, steps, tokens, queue):
    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        total = bench.max_over_ranks(local_ms[rank], torch.device("cpu"))
        value = bench.whole_job_tokens_per_s(world, tokens, total / steps)
        queue.put((rank, total, value))
    finally:
        dist.destroy_process_group()


def _run(world, local_ms, steps, tokens):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, local_ms, steps, tokens, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_two_ranks_take_the_slowest_rank_and_count_all_tokens():
    steps, tokens = 50, 8
    out = _run(2, [12.5, 20.0], steps, tokens)
    for rank, total, value in out:
        assert total == 20.0
        assert value == pytest.approx(2 * tokens / (20.0 / steps * 1e-3))


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench

    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
    assert bench.whole_job_tokens_per_s(1, 8, 0.5) == pytest.approx(16000.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
