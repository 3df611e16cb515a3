"""Multi-rank host logic of the replica runs (`bench.py --gpus N`) on the
CPU: world size 2 over gloo, the ranks as spawned processes (the GPU runs
use the same code over NCCL).  Covered: the barrier, the maximum of the
ranks' times, per-rank data seeds, the whole-job throughput (every rank's
units over the slowest rank's time), a rank that leaves without arriving
(its peer's next collective fails within the timeout instead of hanging),
and the reference arm under torchrun (rank 0 alone works and prints one
line; the other rank exits 0 without output)."""
import json
import os
import queue
import socket
import subprocess
import sys
import time

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from transformer_lm_pretraining_b200.replicas import Replicas

    try:
        r = Replicas("gloo", timeout_s=10)
    except Exception as e:  # pragma: no cover - reported to the test
        q.put((rank, "init failed", repr(e)))
        return
    if mode == "ok":
        r.barrier()
        ms = r.max(10.0 * (rank + 1))  # rank 1 is the slower one
        q.put((rank, ms, r.data_seed(1), r.throughput(1000.0, ms), r.is_root))
        r.close()
    else:  # "absent": rank 1 leaves without arriving at the barrier
        if rank == 1:
            os._exit(0)
        t0 = time.time()
        try:
            r.barrier()
            r.max(1.0)
            q.put((rank, "no error", time.time() - t0))
        except Exception:
            q.put((rank, "raised", time.time() - t0))


def _run(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, world, port, q, mode)) for i in range(world)]
    for p in procs:
        p.start()
    out = []
    deadline = time.time() + 90
    expected = world if mode == "ok" else 1
    while len(out) < expected and time.time() < deadline:
        try:
            out.append(q.get(timeout=1))
        except queue.Empty:
            pass
    for p in procs:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    return sorted(out)


def test_two_ranks_barrier_max_and_throughput():
    out = _run("ok")
    assert len(out) == 2, out
    (r0, ms0, s0, v0, root0), (r1, ms1, s1, v1, root1) = out
    assert (r0, r1) == (0, 1)
    assert ms0 == ms1 == 20.0  # the slower rank's time on every rank
    assert s0 != s1  # each replica draws its own tokens
    assert v0 == v1 == pytest.approx(2 * 1000.0 / 0.020)  # both ranks' units over 20 ms
    assert root0 and not root1


def test_absent_rank_fails_the_peer_instead_of_hanging():
    out = _run("absent")
    assert len(out) == 1, out
    rank, what, seconds = out[0]
    assert rank == 0 and what == "raised"
    assert seconds < 60


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--workload", "tiny", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
