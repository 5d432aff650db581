"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (one process each), as
torchrun would start them.  The hot path has no collective (every rank runs its own
replica); the ranks only reduce timings with MAX and meet at barriers, and only rank 0
prints the result line."""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as td  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_env()
    bench.init_dist(w, "gloo")
    got = bench.reduce_max(10.0 + 5.0 * r, w)   # per-rank timings 10 and 15
    bench.barrier(w)
    got_min_side = bench.reduce_max(-1.0 - r, w)
    out_q.put((r, got, got_min_side))
    td.barrier()
    td.destroy_process_group()


def test_reduce_max_and_barrier_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert [x[1] for x in res] == [15.0, 15.0]       # every rank sees the max over ranks
    assert [x[2] for x in res] == [-1.0, -1.0]


def test_reference_arm_prints_on_rank_zero_only():
    # bench.py --impl reference under a two-rank torchrun-style launch (gloo, CPU):
    # rank 0 alone times the oracle and prints one JSON line; rank 1 exits 0 silently
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   WORLD_SIZE="2", LOCAL_RANK=str(r))
        procs.append(subprocess.Popen(
            [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
             "--steps", "1", "--warmup", "3", "--ref-budget", "2", "--workload", "tiny_q8_d64"],
            env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=300) for p in procs]
    assert [p.returncode for p in procs] == [0, 0], [o[1][-2000:] for o in outs]
    lines0 = [l for l in outs[0][0].splitlines() if l.startswith("{")]
    assert len(lines0) == 1 and not [l for l in outs[1][0].splitlines() if l.startswith("{")]
    d = json.loads(lines0[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
