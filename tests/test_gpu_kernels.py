"""Kernel-level parity on the GPU: the projection GEMM (every operand layout
and epilogue the step uses) and causal attention forward/backward, each
called through the C ABI (gpt2_kernels.h) and compared element by element
with the CPU oracle on the same bf16-representable inputs.

Tolerances (bf16 build): inputs are exactly representable, products are
accumulated in fp32, so the only sizeable error is the final rounding of a
bf16 output (relative 2^-9) plus fp32 accumulation (~K * 2^-24 relative);
bf16 outputs are checked at |gpu - ref| <= 2^-7 |ref| + 2^-9 rms(ref) and
fp32 outputs at 1e-5 rms(ref).  Attention outputs pass through bf16 P and
bf16 operands of the second product: |gpu - ref| <= 2e-2 rms(ref) + 2^-7|ref|;
the backward also uses D = rowsum(dO * O) of the bf16 forward output, whose
rounding is amplified by the cancellation in dP - D: 5e-2 rms(ref) + 2^-6|ref|.
"""
import numpy as np
import pytest

import oracle
from oracle import Config, Oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402


def bf16(a):
    """Round a float array to bf16 values (returned as fp64 numpy)."""
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).float().double().numpy()


def dev(a, dtype=torch.bfloat16):
    return torch.tensor(np.asarray(a, np.float32), device="cuda").to(dtype).contiguous()


def host(t):
    return t.float().cpu().double().numpy()


def rms(a):
    return float(np.sqrt(np.mean(np.square(a)))) + 1e-30


def assert_bf16_close(got, ref, rel=2 ** -7, frac=2 ** -9):
    err = np.abs(got - ref)
    bound = rel * np.abs(ref) + frac * rms(ref) + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside bound; worst "
                           f"{(err / bound).max():.2f}x at {np.unravel_index(np.argmax(err / bound), err.shape)}")


ORC = Oracle(Config(1, 1, 8, 8, 64, 8))  # shape-free primitives
ORC_MP = Oracle(Config(1, 1, 8, 8, 64, 8), openmp=True)


def ref_linear(x, W, b=None):
    return ORC_MP.linear_fwd(x, W, b)


# (129, 512, 64): a pair tile whose second CTA holds one live row;
# (257, 256, 520): one row past a pair tile, N one tile wide, K ragged
GEMM_SHAPES = [(128, 256, 64), (256, 384, 192), (300, 200, 136), (1000, 768, 768),
               (64, 2304, 768), (513, 50304 // 8, 768), (16384, 768, 64), (129, 512, 64),
               (257, 256, 520)]


@pytest.fixture(params=[1, 0], ids=["pairs", "single"])
def cta_pairs(request):
    """Both tilings of the wide products: 256 x 256 tiles over CTA pairs
    (the default) and 128 x 256 tiles on single CTAs."""
    prev = g2.gpt2k_gemm_set_cta_pairs(request.param)
    yield request.param
    g2.gpt2k_gemm_set_cta_pairs(prev)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("epi", ["store", "bias", "bias_gelu", "bias_resid"])
def test_gemm_forward(M, N, K, epi, cta_pairs):
    rng = np.random.default_rng(M * 7 + N + K)
    x = bf16(rng.standard_normal((M, K)))
    W = bf16(rng.standard_normal((N, K)) * 0.05)
    b = rng.standard_normal(N).astype(np.float32) * 0.1
    r = bf16(rng.standard_normal((M, N)))
    ref = ref_linear(x, W, b.astype(np.float64) if epi != "store" else None)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    aux = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    A, B = dev(x), dev(W)
    bias = torch.tensor(b, device="cuda")
    res = dev(r)
    g2.gpt2k_gemm(epi, M, N, K, A, K, 0, B, K, 0, 1.0, out=out, ldo=N,
                  bias=bias if epi != "store" else None, resid=res if epi == "bias_resid" else None,
                  ldr=N, aux=aux if epi == "bias_gelu" else None, ldaux=N)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    got = host(out)
    if epi == "bias_resid":
        ref = ref + r
    if epi == "bias_gelu":
        assert_bf16_close(host(aux), ref)
        ref = ORC.gelu_tanh(bf16(host(aux)))
    assert_bf16_close(got, ref)


@pytest.mark.parametrize("M,N,K", [(16, 768, 768), (16, 3072, 768), (5, 768, 3072), (128, 200, 520),
                                   (16, 2304, 72)])
@pytest.mark.parametrize("epi", ["store", "bias", "bias_gelu", "bias_resid"])
def test_gemm_small_m_split(M, N, K, epi):
    """A single 128-row tile (one position per sequence, as in generation)
    with a split-K workspace: K is split across the SMs, the fp32 partials
    summed in split order and the bf16 epilogue applied after (alpha 0.5)."""
    rng = np.random.default_rng(M * 11 + N + 3 * K)
    x = bf16(rng.standard_normal((M, K)))
    W = bf16(rng.standard_normal((N, K)) * 0.05)
    b = rng.standard_normal(N).astype(np.float32) * 0.1
    r = bf16(rng.standard_normal((M, N)))
    ref = 0.5 * ref_linear(x, W)
    if epi != "store":
        ref = ref + b.astype(np.float64)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    aux = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(8 * M * N, dtype=torch.float32, device="cuda")
    g2.gpt2k_gemm(epi, M, N, K, dev(x), K, 0, dev(W), K, 0, 0.5, out=out, ldo=N,
                  bias=torch.tensor(b, device="cuda") if epi != "store" else None,
                  resid=dev(r) if epi == "bias_resid" else None, ldr=N,
                  aux=aux if epi == "bias_gelu" else None, ldaux=N, split_ws=ws)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    got = host(out)
    if epi == "bias_resid":
        ref = ref + r
    if epi == "bias_gelu":
        assert_bf16_close(host(aux), ref)
        ref = ORC.gelu_tanh(bf16(host(aux)))
    assert_bf16_close(got, ref)


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 200, 136), (1000, 768, 3072), (256, 3072, 768),
                                   (129, 512, 200)])
@pytest.mark.parametrize("epi", ["store", "dgelu"])
def test_gemm_dgrad(M, N, K, epi, cta_pairs):
    """out[M, N] = dy[M, K] W[K, N] (W read MN-major, as the weight is stored)."""
    rng = np.random.default_rng(M + 3 * N + K)
    dy = bf16(rng.standard_normal((M, K)))
    W = bf16(rng.standard_normal((K, N)) * 0.05)
    u = bf16(rng.standard_normal((M, N)) * 2)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    g2.gpt2k_gemm(epi, M, N, K, dev(dy), K, 0, dev(W), N, 1, 0.5, out=out, ldo=N,
                  aux=dev(u) if epi == "dgelu" else None, ldaux=N)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    ref = 0.5 * ref_linear(dy, np.ascontiguousarray(W.T))
    if epi == "dgelu":
        ref = ref * ORC.gelu_tanh_grad(u)
    assert_bf16_close(host(out), ref)


@pytest.mark.parametrize("M,N,K,split", [(256, 128, 192, False), (200, 136, 300, False),
                                         (768, 768, 4096, True), (2304, 768, 2048, True),
                                         (3072, 768, 1000, True), (1024, 512, 520, False)])
def test_gemm_wgrad_accumulates(M, N, K, split, cta_pairs):
    """out32[M, N] += sum_k dy[k, M] x[k, N]: both operands MN-major (tokens
    are the reduction), fp32 accumulate, optional fixed-order split-K."""
    rng = np.random.default_rng(M + N + 5 * K)
    dy = bf16(rng.standard_normal((K, M)))
    x = bf16(rng.standard_normal((K, N)))
    g0 = rng.standard_normal((M, N)).astype(np.float32)
    out32 = torch.tensor(g0, device="cuda")
    ws = torch.zeros(8 * M * N, dtype=torch.float32, device="cuda") if split else None
    g2.gpt2k_gemm("f32_acc", M, N, K, dev(dy), M, 1, dev(x), N, 1, 0.25, out32=out32, ldo32=N,
                  split_ws=ws)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    ref = g0 + 0.25 * ref_linear(np.ascontiguousarray(dy.T), np.ascontiguousarray(x.T))
    got = out32.cpu().double().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * rms(ref) * np.sqrt(K / 64)


@pytest.mark.parametrize("M,N,K", [(1000, 768, 768), (16384, 3072, 768)])
def test_gemm_forward_is_deterministic(M, N, K, cta_pairs):
    rng = np.random.default_rng(M + N)
    A = dev(bf16(rng.standard_normal((M, K))))
    B = dev(bf16(rng.standard_normal((N, K)) * 0.05))
    bias = torch.tensor(rng.standard_normal(N).astype(np.float32), device="cuda")
    outs = []
    for _ in range(2):
        o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        u = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        g2.gpt2k_gemm("bias_gelu", M, N, K, A, K, 0, B, K, 0, 1.0, out=o, ldo=N, bias=bias,
                      aux=u, ldaux=N)
        outs.append((o.view(torch.int16).cpu().numpy(), u.view(torch.int16).cpu().numpy()))
    assert g2.gpt2k_take_error() == 0
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("form", ["dgrad", "bias_resid", "wgrad"])
def test_gemm_pairs_match_single_ctas(form):
    """The two tilings accumulate every output in the same k order, so they
    agree bit for bit."""
    rng = np.random.default_rng(17)
    M, N, K = 1000, 768, 3072
    outs = []
    for pairs in (1, 0):
        prev = g2.gpt2k_gemm_set_cta_pairs(pairs)
        if form == "dgrad":
            dy = dev(bf16(np.random.default_rng(1).standard_normal((M, K))))
            W = dev(bf16(np.random.default_rng(2).standard_normal((K, N)) * 0.05))
            o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            g2.gpt2k_gemm("store", M, N, K, dy, K, 0, W, N, 1, 0.5, out=o, ldo=N)
            outs.append(o.view(torch.int16).cpu().numpy())
        elif form == "bias_resid":
            x = dev(bf16(np.random.default_rng(3).standard_normal((M, K))))
            W = dev(bf16(np.random.default_rng(4).standard_normal((N, K)) * 0.05))
            r = dev(bf16(np.random.default_rng(5).standard_normal((M, N))))
            b = torch.tensor(np.random.default_rng(6).standard_normal(N).astype(np.float32), device="cuda")
            o = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            g2.gpt2k_gemm("bias_resid", M, N, K, x, K, 0, W, K, 0, 1.0, out=o, ldo=N, bias=b,
                          resid=r, ldr=N)
            outs.append(o.view(torch.int16).cpu().numpy())
        else:  # weight gradient without split-K: M = 768 output rows, tokens reduced
            dy = dev(bf16(np.random.default_rng(7).standard_normal((K, N))))
            x = dev(bf16(np.random.default_rng(8).standard_normal((K, 512))))
            o = torch.zeros((N, 512), dtype=torch.float32, device="cuda")
            g2.gpt2k_gemm("f32_acc", N, 512, K, dy, N, 1, x, 512, 1, 1.0, out32=o, ldo32=512)
            outs.append(o.cpu().numpy())
        g2.gpt2k_gemm_set_cta_pairs(prev)
    assert g2.gpt2k_take_error() == 0
    assert np.array_equal(outs[0], outs[1])


def test_gemm_is_deterministic():
    rng = np.random.default_rng(9)
    M, N, K = 768, 768, 4096
    dy, x = dev(bf16(rng.standard_normal((K, M)))), dev(bf16(rng.standard_normal((K, N))))
    ws = torch.zeros(8 * M * N, dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(2):
        o = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        g2.gpt2k_gemm("f32_acc", M, N, K, dy, M, 1, x, N, 1, 1.0, out32=o, ldo32=N, split_ws=ws)
        outs.append(o.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


# head dims 32 / 64 / 128; for head dim 64 (the tensor-core kernels): one
# ragged tile, one full tile, an odd tile count (a query-tile pair without
# its second tile), more work items than SMs, and the training shape
ATTN_SHAPES = [(1, 64, 64, 2), (2, 200, 128, 2), (2, 130, 256, 2), (1, 77, 128, 4),
               (2, 64, 128, 2), (3, 128, 64, 1), (1, 300, 128, 2), (16, 256, 768, 12),
               (2, 1024, 768, 12)]


def _attn_inputs(B, T, C, H, seed):
    rng = np.random.default_rng(seed)
    qkv = bf16(rng.standard_normal((B * T, 3 * C)))
    datt = bf16(rng.standard_normal((B * T, C)))
    return qkv, datt


@pytest.mark.parametrize("B,T,C,H", ATTN_SHAPES)
def test_attention_forward_backward(B, T, C, H):
    o = Oracle(Config(1, H, C, 8, 64, T), openmp=True)
    qkv, datt = _attn_inputs(B, T, C, H, B * T + C)
    ref_y = o.attention_fwd(qkv, B, T)
    att = torch.zeros((B * T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    q = dev(qkv)
    g2.gpt2k_attention_fwd(att, lse, q, B, T, C, H)
    torch.cuda.synchronize()
    y = host(att)
    assert_bf16_close(y, ref_y, rel=2 ** -7, frac=2e-2)
    # lse: log sum_j exp(q.k_j / sqrt(hd)) over j <= i, checked on a few rows
    hd = C // H
    lse_h = lse.cpu().double().numpy().reshape(B, H, T)
    for (b, h, i) in [(0, 0, 0), (B - 1, H - 1, T - 1), (0, H // 2, T // 2)]:
        qi = qkv[b * T + i, h * hd:(h + 1) * hd]
        ks = qkv[b * T: b * T + i + 1, C + h * hd: C + (h + 1) * hd]
        s = ks @ qi / np.sqrt(hd)
        want = s.max() + np.log(np.exp(s - s.max()).sum())
        assert abs(lse_h[b, h, i] - want) < 1e-3 * max(1.0, abs(want))
    # backward with the GPU's own (bf16) forward output, as in training
    ref_d = o.attention_bwd(qkv, datt, B, T)
    dqkv = torch.zeros((B * T, 3 * C), dtype=torch.bfloat16, device="cuda")
    dsum = torch.zeros(g2.gpt2k_attention_bwd_scratch(B, T, H), dtype=torch.float32, device="cuda")
    g2.gpt2k_attention_bwd(dqkv, dsum, dev(datt), q, att, lse, B, T, C, H)
    torch.cuda.synchronize()
    got = host(dqkv)
    # dQ_i = scale sum_j P_ij (dP_ij - D_i) k_j: the bf16 rounding of O in
    # D_i = sum_d dO_id O_id (|delta D_i| <= 2^-8 sum_d |dO_id O_id|) moves
    # dQ_i by up to scale * |delta D_i| * max_j |k_j| (sum_j P_ij = 1).
    o_bf = host(att)
    dabs = np.abs(datt * o_bf).reshape(B * T, H, hd).sum(-1)
    kmax = np.abs(qkv[:, C:2 * C]).reshape(B, T, H, hd).max(axis=1)
    extra_q = (2 ** -8 / np.sqrt(hd)) * dabs.reshape(B, T, H, 1) * kmax[:, None]
    # dK_j = scale sum_i P_ij (dP_ij - D_i) q_i sums the same D_i errors over
    # the queries attending to key j: |delta dK_jd| <= scale sum_i P_ij
    # |delta D_i| |q_id|, with P the exact causal softmax.  The whole of each
    # part is checked in relative L2 as well.
    extra_k = np.zeros((B, T, H, hd))
    q4 = qkv[:, :C].reshape(B, T, H, hd).astype(np.float64)
    k4 = qkv[:, C:2 * C].reshape(B, T, H, hd).astype(np.float64)
    dD = 2 ** -8 * dabs.reshape(B, T, H)
    causal = np.tril(np.ones((T, T), dtype=bool))
    for bb in range(B):
        for hh in range(H):
            sc = q4[bb, :, hh] @ k4[bb, :, hh].T / np.sqrt(hd)
            sc = np.where(causal, sc, -np.inf)
            pm = np.exp(sc - sc.max(axis=1, keepdims=True))
            pm /= pm.sum(axis=1, keepdims=True)
            extra_k[bb, :, hh] = (pm * dD[bb, :, hh][:, None]).T @ np.abs(q4[bb, :, hh]) / np.sqrt(hd)
    extra = [extra_q.reshape(B * T, C), extra_k.reshape(B * T, C), 0.0]
    frac = [5e-2, 5e-2, 5e-2]
    for part in range(3):
        sl = slice(part * C, (part + 1) * C)
        err = np.abs(got[:, sl] - ref_d[:, sl])
        bound = 2 ** -6 * np.abs(ref_d[:, sl]) + frac[part] * rms(ref_d[:, sl]) + extra[part]
        assert (err <= bound).all(), (part, (err / bound).max())
        assert np.linalg.norm(got[:, sl] - ref_d[:, sl]) <= 1e-2 * np.linalg.norm(ref_d[:, sl])


def test_attention_backward_is_deterministic():
    B, T, C, H = 2, 256, 128, 2
    qkv, datt = _attn_inputs(B, T, C, H, 1)
    q, d = dev(qkv), dev(datt)
    att = torch.zeros((B * T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(B * H * T, dtype=torch.float32, device="cuda")
    g2.gpt2k_attention_fwd(att, lse, q, B, T, C, H)
    outs = []
    for _ in range(2):
        dq = torch.zeros((B * T, 3 * C), dtype=torch.bfloat16, device="cuda")
        ds = torch.zeros(g2.gpt2k_attention_bwd_scratch(B, T, H), dtype=torch.float32, device="cuda")
        g2.gpt2k_attention_bwd(dq, ds, d, q, att, lse, B, T, C, H)
        outs.append(dq.view(torch.int16).cpu().numpy())
    assert np.array_equal(outs[0], outs[1])


def test_bounded_wait_expiry_reports_and_recovers():
    """The bounded waits' abort path, made to run: a GEMM whose TMA producer
    (CTA 0) skips one k-block, so that the MMA issuer's wait for it runs out
    (about 2 s).  The kernel reports ERR_TIMEOUT (bit value 4) in the error
    word, every role leaves, TMEM is freed and the launch completes; the
    next product on the same context is correct and reports nothing."""
    M, N, K = 256, 128, 512  # single-CTA 128 x 128 tiles: a few CTAs, one withholds
    rng = np.random.default_rng(5)
    x = bf16(rng.standard_normal((M, K)))
    w = bf16(rng.standard_normal((N, K)) * 0.05)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    g2.gpt2k_take_error()  # start from a clear error word
    assert g2.gpt2k_gemm_expiry_test(M, N, K, dev(x), dev(w), out, kblock=0) == 0
    torch.cuda.synchronize()  # the launch completes: no hang
    assert g2.gpt2k_take_error() & 4
    out2 = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    g2.gpt2k_gemm("store", M, N, K, dev(x), K, 0, dev(w), K, 0, 1.0, out=out2, ldo=N)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    assert_bf16_close(host(out2), ref_linear(x, w))
