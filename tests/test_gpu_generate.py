"""Autoregressive generation with a key/value cache (gpt2_generate) on the
GPU against the CPU oracle.

Each new token's logits (returned by the call) are compared with the
oracle's full forward over the same prefix, the prefix being the GPU's own
generated sequence, so that one near-tie cannot make the two sequences
diverge.  fp32 validation build: logits within 1e-4 (1 + |ref|), and the
greedy token equals the oracle's argmax wherever its top-2 gap exceeds that
bound.  bf16 build: logits within 3e-2 (1 + |ref|) (the whole-step bf16
tolerance of the loss, per logit).  Sampling: the token equals the oracle
sampler applied to the GPU's own logits (the decision taken in the same
fp32 precision) at the same SplitMix64 draw, lies in the top-k set, and
reruns are identical.
"""
import contextlib

import numpy as np
import pytest

import oracle
from oracle import Config, Oracle
from transformer_lm_pretraining_b200.inputs import iid_batch

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402

CASES = [
    ("hd32", Config(2, 4, 128, 1024, 1024, 64), 2, 5, 24),
    ("hd64_padded", Config(2, 2, 128, 1000, 1024, 160), 3, 7, 40),
]


def run_generate(precision, cfg, B, Tp, Ttot, temperature=0.0, top_k=0, seed=0, stream=False):
    """stream=True runs the model on a stream of its own, where the decode
    steps after the first replay one captured CUDA graph; on the default
    stream every step is plain launches."""
    params = Oracle(cfg).init(0).astype(np.float32)
    prompt, _ = iid_batch(cfg.V, B, Tp, 11)
    tok = np.zeros((B, Ttot), np.int32)
    tok[:, :Tp] = prompt
    td = torch.tensor(tok, device="cuda")
    logits = torch.zeros((Ttot - Tp, B, cfg.V), dtype=torch.float32, device="cuda")
    st = torch.cuda.Stream() if stream else None
    with torch.cuda.stream(st) if stream else contextlib.nullcontext():
        m = g2.GPT2(*cfg.args, seed=0, precision=precision, B=B, T=Tp)
        if stream:
            m.set_stream(st)
        m.set_params(params)
        m.generate(td, Tp, temperature, top_k, seed, step_logits=logits)
        torch.cuda.synchronize()
        m.close()
    return params, td.cpu().numpy(), logits.cpu().numpy()


def oracle_step_logits(cfg, params, tok, Tp, Ttot):
    """The oracle's logits for every generated position, from its full
    forward over the (GPU-generated) prefix."""
    o = Oracle(cfg, openmp=True)
    B = tok.shape[0]
    out = np.zeros((Ttot - Tp, B, cfg.V))
    for p in range(Tp, Ttot):
        _, _, lg = o.forward(params.astype(np.float64), tok[:, :p], None, B, p, want_logits=True)
        out[p - Tp] = lg.reshape(B, p, cfg.V)[:, p - 1]
    return out


@pytest.mark.parametrize("name,cfg,B,Tp,Ttot", CASES)
def test_greedy_generation_fp32_matches_oracle(name, cfg, B, Tp, Ttot):
    params, tok, lg = run_generate("fp32", cfg, B, Tp, Ttot)
    ref = oracle_step_logits(cfg, params, tok, Tp, Ttot)
    tol = 1e-4 * (1.0 + np.abs(ref))
    assert np.all(np.abs(lg - ref) <= tol), np.abs(lg - ref).max()
    for s in range(Ttot - Tp):
        for b in range(B):
            srt = np.sort(ref[s, b])[::-1]
            if srt[0] - srt[1] > 2 * tol[s, b].max():
                assert tok[b, Tp + s] == int(np.argmax(ref[s, b])), (s, b)
            assert tok[b, Tp + s] == int(np.argmax(lg[s, b]))  # greedy on its own logits


@pytest.mark.parametrize("name,cfg,B,Tp,Ttot", CASES)
def test_greedy_generation_bf16_matches_oracle(name, cfg, B, Tp, Ttot):
    params, tok, lg = run_generate("bf16", cfg, B, Tp, Ttot, stream=True)  # graph-replayed decode
    ref = oracle_step_logits(cfg, params, tok, Tp, Ttot)
    assert np.all(np.abs(lg - ref) <= 3e-2 * (1.0 + np.abs(ref))), np.abs(lg - ref).max()
    assert np.array_equal(tok[:, Tp:].T, np.argmax(lg, axis=-1))


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_sampled_generation_matches_oracle_sampler(precision):
    name, cfg, B, Tp, Ttot = CASES[1]
    temp, k, seed = 0.8, 20, 123
    params, tok, lg = run_generate(precision, cfg, B, Tp, Ttot, temp, k, seed)
    _, tok2, _ = run_generate(precision, cfg, B, Tp, Ttot, temp, k, seed)
    assert np.array_equal(tok, tok2)  # reruns are identical
    o32 = Oracle(cfg, np.float32)
    for s in range(Ttot - Tp):
        for b in range(B):
            p = Tp + s
            row = lg[s, b].astype(np.float32)
            assert row[tok[b, p]] >= np.sort(row)[::-1][k - 1]  # inside the top-k set
            u = oracle.sample_uniform(seed, p, b)
            assert tok[b, p] == o32.sample_token(row, temp, k, u), (s, b)


def test_generate_rejects_bad_arguments():
    name, cfg, B, Tp, Ttot = CASES[0]
    m = g2.GPT2(*cfg.args, seed=0, precision="bf16", B=B, T=Tp)
    for tp, tt in ((0, 8), (5, 5), (5, cfg.Tmax + 1)):
        td = torch.zeros((B, max(tt, 1)), dtype=torch.int32, device="cuda")
        with pytest.raises(g2.GPT2Error):
            m.generate(td, tp)
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_graph_replayed_decode_equals_plain_launches(precision):
    """The decode steps replayed from one captured graph (a stream of the
    model's own) give the same tokens and logits, bit for bit, as plain
    launches on the default stream, sampled at temperature 0.8, top-k 40."""
    name, cfg, B, Tp, Ttot = CASES[1]
    _, tok_a, lg_a = run_generate(precision, cfg, B, Tp, Ttot, 0.8, 40, 7, stream=False)
    _, tok_b, lg_b = run_generate(precision, cfg, B, Tp, Ttot, 0.8, 40, 7, stream=True)
    assert np.array_equal(tok_a, tok_b)
    assert np.array_equal(lg_a, lg_b)
