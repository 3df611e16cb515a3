"""The weight-gradient GEMM entry point that allocates nothing
(gpt2k_gemm_wgrad_noalloc).

Some callers keep every byte of device memory under their own allocator --
PyTorch's caching allocator, for one, may already hold nearly all free memory
-- so they can neither hand this library a split-K workspace nor let it call
cudaMalloc.  For them the library keeps one fixed 16 MiB array per GPU.  These
tests call that entry point through the C ABI and check it against the
workspace-taking gpt2k_gemm on two calls in a row (the second call reuses the
array the first one left filled), with the fp32 tolerance of the other GEMM
tests, and check that a size beyond the array is refused up front.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402


def _bf16_dev(a):
    return torch.tensor(np.asarray(a, np.float32), device="cuda").to(torch.bfloat16).contiguous()


def _rms(a):
    return float(np.sqrt(np.mean(np.square(a)))) + 1e-30


def test_noalloc_matches_workspace_gemm_on_two_calls():
    # the first shape's calls pass an error word of their own; the second
    # shape's calls pass none, so a bounded-wait expiry would land in the
    # library's private word, which gpt2k_take_error reads and clears
    g2.gpt2k_take_error()
    for M, N, K, seed, own_err in [(768, 512, 4096, 1, True), (256, 768, 2048, 2, False)]:
        rng = np.random.default_rng(seed)
        dy = _bf16_dev(rng.standard_normal((K, M)))
        x = _bf16_dev(rng.standard_normal((K, N)))
        g0 = rng.standard_normal((M, N)).astype(np.float32)

        want = torch.tensor(g0, device="cuda")
        ws = torch.zeros(8 * M * N, dtype=torch.float32, device="cuda")
        g2.gpt2k_gemm("f32_acc", M, N, K, dy, M, 1, x, N, 1, 0.5, out32=want, ldo32=N, split_ws=ws)
        torch.cuda.synchronize()
        assert g2.gpt2k_take_error() == 0  # the workspace-taking reference call

        err = torch.zeros(1, dtype=torch.int32, device="cuda") if own_err else None
        for call in range(2):  # the second call finds the array as the first left it
            got = torch.tensor(g0, device="cuda")
            rc = g2.gpt2k_gemm_wgrad_noalloc(M, N, K, dy, M, x, N, 0.5, got, N, max_splits=8,
                                             err=err)
            assert rc == 0
            torch.cuda.synchronize()
            if own_err:
                assert int(err.item()) == 0, call
            assert g2.gpt2k_take_error() == 0, call
            w, g = want.cpu().double().numpy(), got.cpu().double().numpy()
            assert np.abs(g - w).max() <= 1e-5 * _rms(w) * np.sqrt(K / 64), call


def test_noalloc_refuses_sizes_beyond_its_array():
    M = N = 2048  # 2 * 2048 * 2048 floats > the 4 Mi-float array
    a = torch.zeros((64, M), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    rc = g2.gpt2k_gemm_wgrad_noalloc(M, N, 64, a, M, a, N, 1.0, out, N, max_splits=2)
    assert rc == -1  # GPT2_ERR_ARG, nothing enqueued
    torch.cuda.synchronize()
    assert float(out.abs().max()) == 0.0
