"""The data-parallel step on the GPU through the real exchange path: the
model's device gradient buffer (gpt2_grads_device) summed by NCCL on the
model's stream.  One GPU here, so the process group has one rank and the sum
is the identity: the step must equal the plain step bit for bit, which checks
the buffer view, the in-place collective and its ordering between backward
and clip.  The two-rank arithmetic is covered on the CPU
(test_data_parallel_gloo.py)."""
import datetime
import os
import socket

import numpy as np
import pytest

from oracle import Config, Oracle
from transformer_lm_pretraining_b200.inputs import iid_batch

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402
from transformer_lm_pretraining_b200.data_parallel import DataParallelStep  # noqa: E402

CFG = Config(2, 2, 128, 1000, 1024, 160)
B, T = 2, 64


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("mode,overlap", [("allreduce", False), ("allreduce", True),
                                          ("zero1", False)])
def test_grads_buffer_and_nccl_step_match_the_plain_step(mode, overlap):
    """allreduce: one NCCL sum of the whole buffer, or (overlap) one per
    layer's gradient ranges on a second stream, each started by the event the
    backward records after that layer; zero1: reduce-scatter, shard norm,
    AdamW on the shard, all-gather of the parameters, bf16 refresh."""
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        stream = torch.cuda.Stream()
        torch.cuda.set_stream(stream)
        params = Oracle(CFG).init(0).astype(np.float32)
        models = []
        for _ in range(2):
            m = g2.GPT2(*CFG.args, seed=0, precision="bf16", B=B, T=T)
            m.set_stream(stream)
            m.set_params(params)
            models.append(m)
        batches = []
        for k in range(2):
            tok, tgt = iid_batch(CFG.V, B, T, 40 + k)
            batches.append((torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")))
        # the plain step
        plain = models[0]
        plain.zero_grad()
        for tok, tgt in batches:
            plain.forward(tok, tgt)
            plain.backward(0.5)
        g_view = plain.grads_tensor().cpu().numpy()
        assert np.array_equal(g_view, plain.get_grads())  # the view is the buffer
        n_plain = plain.grad_norm_clip(1.0)
        plain.adamw_step(1e-3, 0.9, 0.95, 1e-8, 0.1)
        # the data-parallel step with the NCCL collectives forced on
        dp = DataParallelStep(
            models[1], 1, 0, mode=mode, overlap=overlap,
            all_reduce=lambda t: dist.all_reduce(t),
            reduce_scatter=lambda out, t: dist.reduce_scatter_tensor(out, t),
            all_gather=lambda out, shard: dist.all_gather_into_tensor(out, shard))
        n_dp = dp(batches, 1e-3)
        torch.cuda.synchronize()
        dp.close()
        if mode == "zero1":  # the norm from the shard's sum of squares (another summation order)
            assert abs(n_dp - n_plain) <= 1e-6 * n_plain
            assert np.abs(models[1].get_params() - plain.get_params()).max() <= 1e-6
        else:
            assert n_dp == n_plain
            assert np.array_equal(models[1].get_params(), plain.get_params())
        for m in models:
            m.close()
    finally:
        torch.cuda.set_stream(torch.cuda.default_stream())
        dist.destroy_process_group()
