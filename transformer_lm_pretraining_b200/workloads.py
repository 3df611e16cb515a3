"""The named workloads: model shape, batch shape and optimiser schedule.

Shapes follow the pages: the 124M GPT-2 at 16 x 1024 tokens per step
("Let's reproduce GPT-2 (124M)" condensed, section 2) and the 524,288-token
step built by gradient accumulation (section 3); the TinyStories GPT
(L8 H8 C512, B64 x T512) and the small GPT (L4 H4 C256, B64 x T256) of
"TinyStories training"; plus a tiny single-step case for parity.
"""
from __future__ import annotations

from dataclasses import dataclass

@dataclass(frozen=True)
class Workload:
    """A model shape plus a batch shape (the five named workloads below)."""
    name: str
    L: int
    H: int
    C: int
    V: int
    Vp: int
    Tmax: int
    B: int
    T: int
    n_micro: int = 1
    lr_max: float = 6e-4
    warmup: int = 715
    max_steps: int = 19073
    iid: bool = False

    @property
    def tokens_per_step(self) -> int:
        return self.B * self.T * self.n_micro

    def flops_per_token(self) -> float:
        """6 * (weights that enter a matmul) + 6 * L * C * T (causal attention)."""
        n_mm = 12 * self.L * self.C * self.C + self.Vp * self.C
        return 6.0 * n_mm + 6.0 * self.L * self.C * self.T

    def flops_per_token_palm(self) -> float:
        n_mm = 12 * self.L * self.C * self.C + self.Vp * self.C
        return 6.0 * n_mm + 12.0 * self.L * self.C * self.T


WORKLOADS = {
    "tiny": Workload("tiny", L=2, H=4, C=128, V=1024, Vp=1024, Tmax=64, B=4, T=64,
                     lr_max=6e-4, warmup=1, max_steps=1, iid=True),
    "small": Workload("small", L=4, H=4, C=256, V=4096, Vp=4096, Tmax=256, B=64, T=256,
                      lr_max=1e-3, warmup=200, max_steps=14000),
    "tinystories": Workload("tinystories", L=8, H=8, C=512, V=4096, Vp=4096, Tmax=512,
                            B=64, T=512, lr_max=1e-3, warmup=200, max_steps=14000),
    "gpt2_124m": Workload("gpt2_124m", L=12, H=12, C=768, V=50257, Vp=50304, Tmax=1024,
                          B=16, T=1024),
    "gpt2_124m_full": Workload("gpt2_124m_full", L=12, H=12, C=768, V=50257, Vp=50304,
                               Tmax=1024, B=64, T=1024, n_micro=8),
}
