"""Multi-rank logic of bench.py on CPU with world-size-2 gloo.

Sequences are independent, so each rank runs its own batch (weak scaling)
and the only cross-rank steps are a barrier and the max over ranks of the
step time; the whole-job value counts every rank's tokens over that time.
The reference arm runs on rank 0 only; other ranks leave without work.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = [1.0 + rank, 10.0 - 3 * rank, 5.0]      # per-rank ms timings
        got = bench.max_over_ranks(local, dist, torch.device("cpu"))
        dist.barrier()
        value = bench.whole_job_rate(64, world, got[0])
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [2.0, 10.0, 5.0]           # element-wise max over ranks
        assert value == pytest.approx(64 * 2 / 2.0e-3)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.whole_job_rate(64, 1, 1.0) == pytest.approx(64000.0)


def test_reference_arm_other_ranks_do_nothing():
    import bench
    import workloads as W

    class A:
        steps, warmup, ref_seqs, gpus = 1, 0, 1, 2
    # rank 1 returns immediately (no oracle work, no output)
    assert bench.run_reference(A(), W.tiny(), 1) == 0


def test_bench_gpus_flag_spawns_ranks():
    # `bench.py --gpus 2` started without a launcher starts its own two ranks
    # (one process each); the dry run exercises that launch path on CPU ranks
    # over gloo and must report both ranks, never one GPU under a 2-GPU label
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                        "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"),
                        "--gpus", "2", "--dry-run-cpu", "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True,
                       timeout=300, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["dry_run"] is True and rec["value"] is None
    assert rec["n_gpus"] == 2 and rec["ranks_seen"] == 2


def test_bench_rejects_mismatched_world_size():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"),
                        "--gpus", "4", "--dry-run-cpu"], capture_output=True,
                       text=True, timeout=120, env=env, cwd=root)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr
