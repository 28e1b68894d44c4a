"""bench.py's multi-rank plumbing on CPU: two gloo ranks, as torchrun launches them
(RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* in the environment).  The timed total is the
maximum over ranks, every rank draws its own requests, and the barrier releases both."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(ws), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    try:
        r, local, w = bench.init_dist("gloo")
        bench.barrier(w)
        # rank r "measured" 10 + r ms: every rank must report the slowest
        m = bench.reduce_max(10.0 + r, w, "cpu")
        q.put((r, local, w, m, bench.shard_seed(7, r)))
        bench.barrier(w)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max_and_draw_disjoint_requests():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[0] for g in got] == [0, 1] and [g[1] for g in got] == [0, 1]
    assert all(g[2] == 2 for g in got)
    assert all(g[3] == 11.0 for g in got)          # max over ranks, on every rank
    assert got[0][4] != got[1][4]                  # disjoint request seeds


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    r, local, w = bench.init_dist("gloo")
    assert (r, local, w) == (0, 0, 1)
    assert bench.reduce_max(3.5, w, "cpu") == 3.5


@pytest.mark.timeout(180)
def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself (here gloo ranks
    on the CPU, via --check-launch, which runs one collective and no GPU work)."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR",
                                                             "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--check-launch"],
                       capture_output=True, text=True, timeout=170, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["world_size"] == 2 and d["ranks_agreed"] == 2
