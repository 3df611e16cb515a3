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
    """The oracle behind the model interface the data-parallel step uses.
    Its flat buffers carry the library's zero padding to a multiple of 2048
    (the ZeRO-1 shards split the padded length)."""

    def __init__(self):
        sys.path.insert(0, ROOT)
        from oracle import Config, Oracle

        self.o = Oracle(Config(*CFG))
        P = self.o.num_params()
        self.padded_params = (P + 2047) // 2048 * 2048
        self._p = np.zeros(self.padded_params)
        self._p[:P] = self.o.init(0)
        self._g = np.zeros(self.padded_params)
        self.p, self.g = self._p[:P], self._g[:P]
        self.m, self.v = np.zeros(P), np.zeros(P)
        self.t = 0
        self.clip_scale = 1.0
        self._batch = None

    def zero_grad(self):
        self.g[:] = 0.0

    def forward(self, tok, tgt):
        self._batch = (tok, tgt)

    def backward(self, scale):
        tok, tgt = self._batch
        self.o.forward_backward(self.p, tok, tgt, B, T, scale, grads=self.g)

    def grads_tensor(self, padded=False):
        return torch.from_numpy(self._g if padded else self.g)  # shares memory with the buffer

    def params_tensor(self, padded=True):
        return torch.from_numpy(self._p if padded else self.p)

    def grad_sumsq(self, begin, end, out):
        out[0] = float(np.sum(self._g[begin:end] ** 2))

    def clip_from_sumsq(self, sumsq, max_norm):
        n = float(np.sqrt(float(sumsq[0])))
        self.clip_scale = max_norm / (n + 1e-6) if n > max_norm else 1.0
        return n

    def adamw_step_range(self, lr, b1, b2, eps, wd, begin, end):
        # AdamW is elementwise: run it on copies and keep this range only
        self.t += 1
        p, g = self.p.copy(), self.g * self.clip_scale
        m, v = self.m.copy(), self.v.copy()
        self.o.adamw(p, g, m, v, self.t, lr, b1, b2, eps, wd)
        end = min(end, self.p.size)
        self.p[begin:end], self.m[begin:end], self.v[begin:end] = p[begin:end], m[begin:end], v[begin:end]
        self.clip_scale = 1.0

    def refresh_weights(self):
        pass

    def grad_norm_clip(self, max_norm):
        return self.o.clip(self.g, max_norm)

    def adamw_step(self, lr, b1, b2, eps, wd):
        self.t += 1
        self.o.adamw(self.p, self.g, self.m, self.v, self.t, lr, b1, b2, eps, wd)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, mode="allreduce"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from transformer_lm_pretraining_b200.data_parallel import DataParallelStep

    dist.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=60))
    model = OracleReplica()
    if mode == "zero1":
        # gloo has no reduce-scatter: the in-place shard of an all-reduce is
        # the same sum; the all-gather goes through a list of shards
        def reduce_scatter(out, t):
            dist.all_reduce(t)

        def all_gather(out, shard):
            parts = [torch.empty_like(shard) for _ in range(world)]
            dist.all_gather(parts, shard.clone())
            out.copy_(torch.cat(parts))

        step = DataParallelStep(model, world, rank, mode="zero1", reduce_scatter=reduce_scatter,
                                all_gather=all_gather)
    else:
        step = DataParallelStep(model, world)
    norms = []
    for s in range(STEPS):
        mine = _batches(s)[rank::world]  # this rank's micro-batches
        norms.append(step(mine, 1e-3))
    q.put((rank, norms, model.p.copy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["allreduce", "zero1"])
def test_two_rank_data_parallel_equals_full_batch_step(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, mode)) for r in range(2)]
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
