"""Data-parallel training step over replicas of the model.

Every rank holds the whole model and runs the forward and backward of its
own micro-batches with the loss scaled by 1 / (micro-batches x ranks), so
that the sum of the ranks' gradients is the gradient of the mean loss over
the global batch.  This follows the pages' multi-GPU runs, which average the
gradients of per-GPU micro-batches before the update (condensed GPT-2 page,
section 3), and the llm.c page's ZeRO-1 option (optimizer-state sharding).
Two exchanges:

  "allreduce"  one sum all-reduce of the fp32 gradient buffer; then every
               rank applies the same global-norm clip and AdamW, so the
               parameters stay identical.  With overlap=True (GPT2 only) the
               gradients of each layer are all-reduced on a second stream as
               soon as the backward has finished that layer (the model
               records one CUDA event per layer), while the backward of the
               layers below still runs.
  "zero1"      a reduce-scatter of the (zero-padded) gradient buffer gives
               each rank the summed gradient of its contiguous shard; the
               global norm is the square root of the all-reduced sum of the
               shards' sums of squares; each rank runs AdamW on its shard of
               the parameters only; an all-gather of the updated fp32
               parameters and a refresh of the bf16 weight copy make the
               replicas identical again.  The communication volume equals one
               all-reduce; the optimizer arithmetic is 1/R per rank.

The model is duck-typed:
    zero_grad(), forward(tok, tgt), backward(loss_scale),
    grads_tensor(padded=False) -> a tensor the collectives work on in place,
    grad_norm_clip(max_norm) -> the pre-clip norm,
    adamw_step(lr, b1, b2, eps, wd),
and for "zero1":
    padded_params, params_tensor(padded=True), grad_sumsq(begin, end, out),
    clip_from_sumsq(sumsq, max_norm) -> the norm,
    adamw_step_range(lr, b1, b2, eps, wd, begin, end), refresh_weights().
GPT2 (device buffers, NCCL on the model's stream) and the CPU oracle of the
tests (gloo) both fit.  With GPT2 the model's stream must be torch's current
stream (GPT2.set_stream and torch.cuda.set_stream), so that the collectives
are ordered after the backward kernels and before the clip.
"""
from __future__ import annotations


def layer_buckets(model):
    """Flat-parameter ranges [(begin, end), ...] per gradient bucket: bucket
    l < L holds layer l's slice of every per-layer tensor, bucket L the
    tensors shared by all positions (wte, wpe, lnf_g, lnf_b)."""
    L = model.cfg[0]
    buckets = [[] for _ in range(L + 1)]
    for name, shape, off in model.tensors():
        numel = 1
        for d in shape:
            numel *= int(d)
        if name in ("wte", "wpe", "lnf_g", "lnf_b"):
            buckets[L].append((off, off + numel))
        else:
            per = numel // L
            for l in range(L):
                buckets[l].append((off + l * per, off + (l + 1) * per))
    return buckets


class DataParallelStep:
    def __init__(self, model, world: int, rank: int = 0, mode: str = "allreduce",
                 overlap: bool = False, all_reduce=None, reduce_scatter=None, all_gather=None,
                 sync: bool = True):
        """all_reduce(t): sum over the ranks in place; reduce_scatter(out, t):
        out = this rank's shard of the sum of every rank's t; all_gather(out,
        shard): out = the ranks' shards in rank order.  The defaults (world >
        1) are torch.distributed's collectives on the default group; given
        callables run even on one rank.  sync=False (GPT2) reads neither the
        loss nor the norm back, so the host can run ahead of the GPU; the step
        then returns None."""
        self.sync = bool(sync)
        if mode not in ("allreduce", "zero1"):
            raise ValueError(mode)
        self.model = model
        self.world = int(world)
        self.rank = int(rank)
        self.mode = mode
        self.overlap = bool(overlap) and mode == "allreduce"
        if self.world > 1:
            import torch.distributed as dist

            if all_reduce is None:
                def all_reduce(t):
                    dist.all_reduce(t, op=dist.ReduceOp.SUM)
            if reduce_scatter is None:
                def reduce_scatter(out, t):
                    dist.reduce_scatter_tensor(out, t, op=dist.ReduceOp.SUM)
            if all_gather is None:
                def all_gather(out, shard):
                    dist.all_gather_into_tensor(out, shard)
        self._all_reduce = all_reduce
        self._reduce_scatter = reduce_scatter
        self._all_gather = all_gather
        self._events = None
        if self.overlap:
            self._setup_overlap()

    # -- bucketed all-reduce overlapped with the backward (GPT2) ----------
    def _setup_overlap(self):
        import torch

        m = self.model
        self._buckets = layer_buckets(m)
        self._comm = torch.cuda.Stream()
        self._events = [torch.cuda.Event() for _ in self._buckets]
        for e in self._events:  # the handles exist once recorded
            e.record()
        m.set_backward_events(self._events)

    def _overlapped_exchange(self):
        import torch

        grads = self.model.grads_tensor()
        L = len(self._buckets) - 1
        main = torch.cuda.current_stream()
        with torch.cuda.stream(self._comm):
            for b in list(range(L - 1, -1, -1)) + [L]:  # the order the backward finishes them
                self._comm.wait_event(self._events[b])
                if self._all_reduce is not None:
                    for lo, hi in self._buckets[b]:
                        self._all_reduce(grads[lo:hi])
        main.wait_stream(self._comm)

    # -- the step ---------------------------------------------------------
    def __call__(self, batches, lr, max_norm=1.0, b1=0.9, b2=0.95, eps=1e-8, wd=0.1):
        """One optimizer step over this rank's micro-batches [(tok, tgt), ...]
        (every rank passes the same number).  Returns the gradient norm before
        clipping, as every rank sees it."""
        m = self.model
        kw = {} if self.sync else {"sync": False}
        m.zero_grad()
        scale = 1.0 / (len(batches) * self.world)
        for tok, tgt in batches:
            if self.sync:
                m.forward(tok, tgt)
            else:
                m.forward(tok, tgt, sync_loss=False)
            m.backward(scale)
        if self.mode == "zero1":
            return self._zero1_update(lr, max_norm, b1, b2, eps, wd, kw)
        if self.overlap:
            self._overlapped_exchange()
        elif self._all_reduce is not None:
            self._all_reduce(m.grads_tensor())
        norm = m.grad_norm_clip(max_norm, **kw)
        m.adamw_step(lr, b1, b2, eps, wd)
        return norm

    def shard(self):
        """This rank's contiguous range of the padded flat buffers."""
        n = self.model.padded_params // self.world
        return self.rank * n, (self.rank + 1) * n

    def _zero1_update(self, lr, max_norm, b1, b2, eps, wd, kw):
        m = self.model
        lo, hi = self.shard()
        grads = m.grads_tensor(padded=True)
        if self._reduce_scatter is not None:
            self._reduce_scatter(grads[lo:hi], grads)  # in place: this rank's shard of the sum
        sumsq = grads.new_zeros(1, dtype=__import__("torch").float64)
        m.grad_sumsq(lo, hi, sumsq)
        if self._all_reduce is not None:
            self._all_reduce(sumsq)
        norm = m.clip_from_sumsq(sumsq, max_norm, **kw)
        m.adamw_step_range(lr, b1, b2, eps, wd, lo, hi)
        params = m.params_tensor(padded=True)
        if self._all_gather is not None:
            self._all_gather(params, params[lo:hi])  # in place
        m.refresh_weights()
        return norm

    def close(self):
        if self._events is not None:
            self.model.set_backward_events(None)
            self._events = None
