"""Replica plumbing for multi-GPU runs of the one-GPU training step.

One process per GPU, started by torch.distributed.run (RANK, LOCAL_RANK,
WORLD_SIZE, MASTER_ADDR/PORT from the environment).  Every rank runs the
whole step on its own data: the step has no exchange between GPUs, so no
gradient, activation or parameter ever crosses ranks.  The only cross-rank
operations are the barriers around a timed region and the maximum of the
ranks' device times; the job's throughput is the units all ranks processed
over that maximum.  Backend: NCCL between GPUs, gloo on the CPU (tests).
A rank that fails or never arrives ends its peers' next barrier with an
error after `timeout_s`.
"""
from __future__ import annotations

import datetime
import os


class Replicas:
    def __init__(self, backend: str = "nccl", timeout_s: float = 120.0, group: bool = False):
        """group=True starts the process group even on one rank (for the
        data-parallel step, whose collectives then run as one-rank NCCL
        calls)."""
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self._dist = None
        if self.world > 1 or group:
            import torch.distributed as dist

            if self.world == 1:
                os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
                if "MASTER_PORT" not in os.environ:
                    import socket

                    with socket.socket() as s:
                        s.bind(("127.0.0.1", 0))
                        os.environ["MASTER_PORT"] = str(s.getsockname()[1])
            dist.init_process_group(backend, rank=self.rank, world_size=self.world,
                                    timeout=datetime.timedelta(seconds=timeout_s))
            self._dist = dist

    @property
    def is_root(self) -> bool:
        return self.rank == 0

    def data_seed(self, base: int = 1) -> int:
        """Each replica draws its own token stream."""
        return base + self.rank

    def barrier(self) -> None:
        if self._dist is not None:
            self._dist.barrier()

    def max(self, x: float) -> float:
        """The maximum of x over the ranks (x itself on one rank)."""
        if self._dist is None:
            return float(x)
        import torch

        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        self._dist.all_reduce(t, op=self._dist.ReduceOp.MAX)
        return float(t.item())

    def throughput(self, units_per_rank: float, ms_max: float) -> float:
        """Whole-job rate: every rank's units over the slowest rank's time."""
        return units_per_rank * self.world / (ms_max / 1e3)

    def close(self) -> None:
        if self._dist is not None:
            self._dist.barrier()
            self._dist.destroy_process_group()
            self._dist = None
