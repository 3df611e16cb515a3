"""Seeded synthetic token streams for the GPT-2 step.

The pages train on FineWeb / FineWeb-Edu (GPT-2 124M) and TinyStories (the
small GPTs); none of those datasets is available here, so every workload runs
on a synthetic Zipf-distributed token stream of the same shape:
p(id) proportional to (id + 1) ** -s over ids 0 .. V-1, with s = 1.1.

This module is the only code shared by the CUDA path's harnesses and by the
CPU oracle's harnesses.  It holds no part of the model's arithmetic: it draws
integers and nothing else.

Definition (so both sides can reproduce it): uniforms are numpy's
``Generator(PCG64(SeedSequence([seed, stream])))``.random() doubles; a token is
the first id whose cumulative probability (float64, normalised so the last
entry is exactly 1) exceeds the uniform.
"""
from __future__ import annotations

from functools import lru_cache

import numpy as np

ZIPF_S = 1.1
DATA_STREAM = 0xDA7A  # keeps data draws apart from every other use of `seed`


@lru_cache(maxsize=8)
def zipf_cdf(V: int, s: float = ZIPF_S) -> np.ndarray:
    w = (np.arange(1, V + 1, dtype=np.float64)) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    cdf[-1] = 1.0
    return cdf


def zipf_draw(rng: np.random.Generator, n: int, V: int, s: float = ZIPF_S) -> np.ndarray:
    u = rng.random(n)
    ids = np.searchsorted(zipf_cdf(V, s), u, side="right")
    return np.minimum(ids, V - 1).astype(np.int32)


def make_rng(seed: int, stream: int = DATA_STREAM) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def iid_batch(V: int, B: int, T: int, seed: int = 0):
    """Tokens and targets drawn independently (the tiny single-step case)."""
    rng = make_rng(seed)
    tok = zipf_draw(rng, B * T, V)
    tgt = zipf_draw(rng, B * T, V)
    return tok.reshape(B, T), tgt.reshape(B, T)


class ZipfStream:
    """One long token stream s[0], s[1], ...; chunk j is s[jBT : jBT + BT + 1],
    tokens = chunk[:-1], targets = chunk[1:] (the stream shifted by one)."""

    def __init__(self, V: int, seed: int = 0):
        self.V = V
        self.rng = make_rng(seed)
        self._carry = None

    def next_batch(self, B: int, T: int):
        n = B * T
        if self._carry is None:
            chunk = zipf_draw(self.rng, n + 1, self.V)
        else:
            chunk = np.concatenate([self._carry, zipf_draw(self.rng, n, self.V)])
        self._carry = chunk[-1:].copy()
        return chunk[:-1].reshape(B, T).copy(), chunk[1:].reshape(B, T).copy()
