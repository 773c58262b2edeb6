"""The multi-process paths of bench.py on CPU: world size 2 over gloo.

The operator has no exchange step, so several GPUs run independent replicas;
what several ranks share is the timing protocol (a barrier on both sides of the
timed region, the maximum time over ranks) and, for the reference arm, that
rank 0 alone prints.  Both are checked here without a GPU.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    ranks = bench.Ranks(world, rank, rank, "gloo")
    ranks.barrier()
    t = ranks.max(10.0 + 5.0 * rank)   # a slower rank 1
    ranks.barrier()
    ranks.close()
    q.put((rank, t))


def test_ranks_take_the_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2 and out["steps"] == 2
    assert out["value"] > 0 and out["cpu_baseline"]["kind"] == "oracle"
    assert out["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("world", [1, 2, 4])
def test_value_is_whole_job_throughput(world):
    sys.path.insert(0, ROOT)
    import bench

    # every rank streams the same weights; the job moves world times the bytes
    assert bench.job_gbs(world, 994_635_776, 1.0) == pytest.approx(world * 994.635776)
