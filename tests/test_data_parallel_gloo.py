"""The data-parallel step (transformer_lm_pretraining_b200/data_parallel.py)
on the CPU: two ranks over gloo, each running the oracle on half of a global
batch, against one process running the oracle on the whole batch.  The
all-reduced gradient, the clip norm and the parameters after two AdamW steps
must match the single-process step (up to fp64 summation order), and the two
ranks' parameters must be identical."""
import os
import queue
import socket
import sys
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = (2, 2, 32, 64, 64, 16)  # L, H, C, V, Vpad, Tmax
B, T, N_MICRO, STEPS = 2, 8, 4, 2


def _batches(step):
    from transformer_lm_pretraining_b200.inputs import iid_batch

    out = []
    for k in range(N_MICRO):
        tok, tgt = iid_batch(CFG[3], B, T, 100 * step + k)
        out.append((tok, tgt))
    return out


class OracleReplica:
    """The oracle behind the model interface the data-parallel step uses."""

    def __init__(self):
        sys.path.insert(0, ROOT)
        from oracle import Config, Oracle

        self.o = Oracle(Config(*CFG))
        self.p = self.o.init(0)
        self.g = np.zeros_like(self.p)
        self.m, self.v = np.zeros_like(self.p), np.zeros_like(self.p)
        self.t = 0
        self._batch = None

    def zero_grad(self):
        self.g[:] = 0.0

    def forward(self, tok, tgt):
        self._batch = (tok, tgt)

    def backward(self, scale):
        tok, tgt = self._batch
        self.o.forward_backward(self.p, tok, tgt, B, T, scale, grads=self.g)

    def grads_tensor(self):
        return torch.from_numpy(self.g)  # shares memory: the all-reduce writes self.g

    def grad_norm_clip(self, max_norm):
        return self.o.clip(self.g, max_norm)

    def adamw_step(self, lr, b1, b2, eps, wd):
        self.t += 1
        self.o.adamw(self.p, self.g, self.m, self.v, self.t, lr, b1, b2, eps, wd)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from transformer_lm_pretraining_b200.data_parallel import DataParallelStep

    dist.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=60))
    model = OracleReplica()
    step = DataParallelStep(model, world)
    norms = []
    for s in range(STEPS):
        mine = _batches(s)[rank::world]  # this rank's micro-batches
        norms.append(step(mine, 1e-3))
    q.put((rank, norms, model.p.copy()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_data_parallel_equals_full_batch_step():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = []
    deadline = time.time() + 120
    while len(out) < 2 and time.time() < deadline:
        try:
            out.append(q.get(timeout=1))
        except queue.Empty:
            pass
    for p in procs:
        p.join(timeout=30)
        if p.is_alive():
            p.kill()
    assert len(out) == 2, out
    out.sort(key=lambda x: x[0])
    # single process, whole batch, same schedule
    ref = OracleReplica()
    ref_norms = []
    for s in range(STEPS):
        ref.zero_grad()
        for tok, tgt in _batches(s):
            ref.forward(tok, tgt)
            ref.backward(1.0 / N_MICRO)
        ref_norms.append(ref.grad_norm_clip(1.0))
        ref.adamw_step(1e-3, 0.9, 0.95, 1e-8, 0.1)
    (_, n0, p0), (_, n1, p1) = out
    assert np.array_equal(p0, p1)  # the replicas stay identical
    assert n0 == n1
    np.testing.assert_allclose(n0, ref_norms, rtol=1e-12)
    np.testing.assert_allclose(p0, ref.p, rtol=0, atol=1e-9)
    assert not np.allclose(p0, OracleReplica().p)  # the steps did move the parameters
