"""The multi-rank path of bench.py on CPU (gloo, world size 2): one process per
rank, the barrier, max-over-ranks timing and the whole-job value; and the
reference arm under 2 ranks (rank 0 alone runs and prints)."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws)
    import bench
    bench._barrier(ws)
    ms = 3.0 + rank                          # rank 1 is the slow one
    worst = bench._max_over_ranks(ms, ws)
    value = bench.whole_job_value(2.0e12, ws, worst)
    out.put((rank, worst, value))
    bench._barrier(ws)
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_whole_job_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, worst, value in res:
        assert worst == 4.0                  # both ranks see the slowest rank's time
        assert abs(value - 2 * 2.0e12 / 4.0e-3 / 1e12) < 1e-9


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    if rank == 1:
        assert lines == []
    else:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
        assert d["cpu_baseline"]["kind"] == "oracle"
