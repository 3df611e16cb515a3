"""Run and time single kernels of the step through the kernel-level C ABI.

  python -m transformer_lm_pretraining_b200.kernel_bench gemm --M 16384 --N 3072 --K 768 \
      --form fwd --epi bias_gelu --iters 20
  python -m transformer_lm_pretraining_b200.kernel_bench attn --B 16 --T 1024 --C 768 --H 12

GEMM forms (the three products of a projection y = x W^T + b):
  fwd    out[M, N] = x[M, K] W[N, K]^T            (epi: store, bias, bias_gelu, bias_resid)
  dgrad  out[M, N] = dy[M, K] W[K, N]             (epi: store, dgelu)
  wgrad  out32[M, N] += dy[K, M]^T x[K, N]        (fp32 accumulate, split-K when few tiles)
  python -m transformer_lm_pretraining_b200.kernel_bench ln --M 16384 --C 768 --form bwd
  python -m transformer_lm_pretraining_b200.kernel_bench cls --M 16384 --V 50257 --Vp 50304
Prints one JSON line with the mean time per call (CUDA events, after one
warm-up call) and the achieved TFLOP/s (GEMM, attention) or GB/s of
algorithmic traffic (LayerNorm, classifier).  Inputs are random bf16.
"""
from __future__ import annotations

import argparse
import json

import torch

from transformer_lm_pretraining_b200 import gpt2 as g2


def _rand(shape, scale=1.0):
    return (torch.randn(shape, device="cuda") * scale).to(torch.bfloat16)


def bench_gemm(a):
    M, N, K = a.M, a.N, a.K
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    if a.form == "fwd":
        A, B = _rand((M, K)), _rand((N, K), 0.05)
        bias = torch.randn(N, device="cuda") * 0.1
        resid = _rand((M, N))
        aux = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

        def call():
            g2.gpt2k_gemm(a.epi, M, N, K, A, K, 0, B, K, 0, 1.0, out=out, ldo=N,
                          bias=None if a.epi == "store" else bias,
                          resid=resid if a.epi == "bias_resid" else None, ldr=N,
                          aux=aux if a.epi == "bias_gelu" else None, ldaux=N)
    elif a.form == "dgrad":
        A, B = _rand((M, K)), _rand((K, N), 0.05)
        aux = _rand((M, N))

        def call():
            g2.gpt2k_gemm(a.epi, M, N, K, A, K, 0, B, N, 1, 1.0, out=out, ldo=N,
                          aux=aux if a.epi == "dgelu" else None, ldaux=N)
    else:
        A, B = _rand((K, M)), _rand((K, N))
        out32 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        ws = torch.empty(8 * M * N, dtype=torch.float32, device="cuda")

        def call():
            g2.gpt2k_gemm("f32_acc", M, N, K, A, M, 1, B, N, 1, 1.0, out32=out32, ldo32=N,
                          split_ws=ws)
    return call, 2.0 * M * N * K


def bench_attn(a):
    B, T, C, H = a.B, a.T, a.C, a.H
    qkv = _rand((B * T, 3 * C))
    att = torch.empty((B * T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B * H * T, dtype=torch.float32, device="cuda")
    hd = C // H
    tri = B * H * T * (T + 1) / 2 * hd
    if a.form == "bwd":
        g2.gpt2k_attention_fwd(att, lse, qkv, B, T, C, H)
        datt = _rand((B * T, C))
        dqkv = torch.empty((B * T, 3 * C), dtype=torch.bfloat16, device="cuda")
        dsum = torch.empty(g2.gpt2k_attention_bwd_scratch(B, T, H), dtype=torch.float32, device="cuda")

        def call():
            g2.gpt2k_attention_bwd(dqkv, dsum, datt, qkv, att, lse, B, T, C, H)
        return call, 10.0 * tri

    def call():
        g2.gpt2k_attention_fwd(att, lse, qkv, B, T, C, H)
    return call, 4.0 * tri


def bench_ln(a):
    M, C = a.M, a.C
    x, dy = _rand((M, C)), _rand((M, C))
    g = torch.ones(C, device="cuda")
    b = torch.zeros(C, device="cuda")
    y = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(M, dtype=torch.float32, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    g2.gpt2k_layernorm_fwd(y, mean, rstd, x, g, b, M, C)
    if a.form == "fwd":
        def call():
            g2.gpt2k_layernorm_fwd(y, mean, rstd, x, g, b, M, C)
        return call, 4.0 * M * C + 8.0 * M  # bytes: read x, write y, mean, rstd
    dx = _rand((M, C))
    dg, db, ds = (torch.zeros(C, device="cuda") for _ in range(3))
    part = torch.empty(g2.gpt2k_layernorm_bwd_scratch(C), dtype=torch.float32, device="cuda")

    def call():
        g2.gpt2k_layernorm_bwd(dx, dy, x, mean, rstd, g, dg, db, ds, part, M, C, 1)
    return call, 8.0 * M * C + 8.0 * M  # bytes: read x, dy, dx; write dx; mean, rstd


def bench_cls(a):
    M, V, Vp = a.M, a.V, a.Vp
    z = _rand((M, Vp))
    losses = torch.empty(M, dtype=torch.float32, device="cuda")
    tgt = torch.randint(0, V, (M,), dtype=torch.int32, device="cuda")

    def call():
        g2.gpt2k_classifier(z, losses, tgt, M, V, Vp, write_grad=True)
    return call, 4.0 * M * Vp  # bytes: read and write the logits


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="kind", required=True)
    g = sub.add_parser("gemm")
    g.add_argument("--M", type=int, default=16384)
    g.add_argument("--N", type=int, default=3072)
    g.add_argument("--K", type=int, default=768)
    g.add_argument("--form", default="fwd", choices=["fwd", "dgrad", "wgrad"])
    g.add_argument("--epi", default="bias")
    g.add_argument("--iters", type=int, default=20)
    g.add_argument("--pairs", type=int, default=1, help="256 x 256 tiles over CTA pairs (1) or not (0)")
    t = sub.add_parser("attn")
    t.add_argument("--B", type=int, default=16)
    t.add_argument("--T", type=int, default=1024)
    t.add_argument("--C", type=int, default=768)
    t.add_argument("--H", type=int, default=12)
    t.add_argument("--form", default="fwd", choices=["fwd", "bwd"])
    t.add_argument("--iters", type=int, default=20)
    n = sub.add_parser("ln")
    n.add_argument("--M", type=int, default=16384)
    n.add_argument("--C", type=int, default=768)
    n.add_argument("--form", default="bwd", choices=["fwd", "bwd"])
    n.add_argument("--iters", type=int, default=20)
    c = sub.add_parser("cls")
    c.add_argument("--M", type=int, default=16384)
    c.add_argument("--V", type=int, default=50257)
    c.add_argument("--Vp", type=int, default=50304)
    c.add_argument("--iters", type=int, default=5)
    c.set_defaults(form="fwd+grad")
    a = ap.parse_args()
    torch.manual_seed(0)
    if a.kind == "gemm":
        g2.gpt2k_gemm_set_cta_pairs(a.pairs)
    call, work = {"gemm": bench_gemm, "attn": bench_attn, "ln": bench_ln, "cls": bench_cls}[a.kind](a)
    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    err = g2.gpt2k_take_error()
    rate = ({"gbs": work / (ms / 1e3) / 1e9} if a.kind in ("ln", "cls")
            else {"tflops": work / (ms / 1e3) / 1e12})
    print(json.dumps({"kernel": a.kind, "form": a.form, "args": vars(a), "ms": ms, **rate,
                      "error_word": err}))
    if err:
        raise SystemExit(f"kernel error word {err}")


if __name__ == "__main__":
    main()
