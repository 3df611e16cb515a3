"""Run and time single kernels of the step through the kernel-level C ABI.

  python -m transformer_lm_pretraining_b200.kernel_bench gemm --M 16384 --N 3072 --K 768 \
      --form fwd --epi bias_gelu --iters 20
  python -m transformer_lm_pretraining_b200.kernel_bench attn --B 16 --T 1024 --C 768 --H 12

GEMM forms (the three products of a projection y = x W^T + b):
  fwd    out[M, N] = x[M, K] W[N, K]^T            (epi: store, bias, bias_gelu, bias_resid)
  dgrad  out[M, N] = dy[M, K] W[K, N]             (epi: store, dgelu)
  wgrad  out32[M, N] += dy[K, M]^T x[K, N]        (fp32 accumulate, split-K when few tiles)
Prints one JSON line with the mean time per call (CUDA events, after one
warm-up call) and the achieved TFLOP/s.  Inputs are random bf16.
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
        dsum = torch.empty(B * H * T, dtype=torch.float32, device="cuda")

        def call():
            g2.gpt2k_attention_bwd(dqkv, dsum, datt, qkv, att, lse, B, T, C, H)
        return call, 10.0 * tri

    def call():
        g2.gpt2k_attention_fwd(att, lse, qkv, B, T, C, H)
    return call, 4.0 * tri


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
    t = sub.add_parser("attn")
    t.add_argument("--B", type=int, default=16)
    t.add_argument("--T", type=int, default=1024)
    t.add_argument("--C", type=int, default=768)
    t.add_argument("--H", type=int, default=12)
    t.add_argument("--form", default="fwd", choices=["fwd", "bwd"])
    t.add_argument("--iters", type=int, default=20)
    a = ap.parse_args()
    torch.manual_seed(0)
    call, flops = bench_gemm(a) if a.kind == "gemm" else bench_attn(a)
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
    print(json.dumps({"kernel": a.kind, "form": a.form, "args": vars(a), "ms": ms,
                      "tflops": flops / (ms / 1e3) / 1e12, "error_word": err}))
    if err:
        raise SystemExit(f"kernel error word {err}")


if __name__ == "__main__":
    main()
