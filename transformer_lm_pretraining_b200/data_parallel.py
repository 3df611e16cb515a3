"""Data-parallel training step over replicas of the model.

Every rank holds the whole model and runs the forward and backward of its
own micro-batches with the loss scaled by 1 / (micro-batches x ranks).  The
ranks then sum their fp32 gradient buffers with one all-reduce, and every
rank applies the same global-norm clip and AdamW step, so their parameters
stay identical.  This follows the pages' multi-GPU runs, which average the
gradients of per-GPU micro-batches before the update.  Sharding the
optimizer state (ZeRO-1) is not built.

The model is duck-typed:
    zero_grad(), forward(tok, tgt), backward(loss_scale),
    grads_tensor()  -> a torch tensor the collective sums in place,
    grad_norm_clip(max_norm) -> the pre-clip norm,
    adamw_step(lr, b1, b2, eps, wd).
GPT2 (its device buffer, summed over NCCL on the model's stream) and the CPU
oracle of the tests (gloo) both fit.  With GPT2 the model's stream must be
torch's current stream (GPT2.set_stream and torch.cuda.set_stream), so that
the all-reduce is ordered after the backward kernels and before the clip.
"""
from __future__ import annotations


class DataParallelStep:
    def __init__(self, model, world: int, all_reduce=None):
        """all_reduce(tensor) sums a tensor over the ranks in place; the
        default (for world > 1) is torch.distributed.all_reduce (SUM) on the
        default group.  A given all_reduce runs even on one rank."""
        self.model = model
        self.world = int(world)
        if all_reduce is None and self.world > 1:
            import torch.distributed as dist

            def all_reduce(t):
                dist.all_reduce(t, op=dist.ReduceOp.SUM)
        self._all_reduce = all_reduce

    def __call__(self, batches, lr, max_norm=1.0, b1=0.9, b2=0.95, eps=1e-8, wd=0.1):
        """One optimizer step over this rank's micro-batches [(tok, tgt), ...]
        (every rank passes the same number).  Returns the gradient norm before
        clipping, as every rank sees it."""
        m = self.model
        m.zero_grad()
        scale = 1.0 / (len(batches) * self.world)
        for tok, tgt in batches:
            m.forward(tok, tgt)
            m.backward(scale)
        if self._all_reduce is not None:
            self._all_reduce(m.grads_tensor())
        norm = m.grad_norm_clip(max_norm)
        m.adamw_step(lr, b1, b2, eps, wd)
        return norm
