"""Kernel-level parity on the GPU for the LayerNorm forward/backward and the
softmax cross-entropy (classifier), called through the C ABI
(gpt2_kernels.h) and compared element by element with the CPU oracle on the
same bf16-representable inputs.

Tolerances (bf16 build): statistics and sums are fp32 over bf16 inputs, so
the sizeable error of a bf16 output is its final rounding (relative 2^-9):
bf16 outputs are checked at |gpu - ref| <= 2^-7 |ref| + 2^-9 rms(ref);
fp32 column sums of M terms at 1e-5 of the sum of the terms' magnitudes;
per-row losses (fp32 log-sum-exp over at most 65536 classes with the
hardware exp2, relative error ~2^-22 per term) at 1e-5 (1 + |lse|).
"""
import numpy as np
import pytest

from oracle import Config, Oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402

ORC = Oracle(Config(1, 1, 8, 8, 64, 8), openmp=True)  # shape-free primitives


def bf16(a):
    return torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16).float().double().numpy()


def dev(a, dtype=torch.bfloat16):
    return torch.tensor(np.asarray(a, np.float32), device="cuda").to(dtype).contiguous()


def host(t):
    return t.float().cpu().double().numpy()


def rms(a):
    return float(np.sqrt(np.mean(np.square(a)))) + 1e-30


def assert_close(got, ref, rel, floor):
    err = np.abs(got - ref)
    bound = rel * np.abs(ref) + floor + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside bound; worst "
                           f"{(err / bound).max():.2f}x at "
                           f"{np.unravel_index(np.argmax(err / bound), err.shape)}")


LN_SHAPES = [(1, 8), (37, 64), (300, 520), (4096, 768), (70, 2048)]


def _ln_inputs(M, C, seed):
    rng = np.random.default_rng(seed)
    x = bf16(0.5 + 2.0 * rng.standard_normal((M, C)))
    g = (1.0 + 0.3 * rng.standard_normal(C)).astype(np.float32).astype(np.float64)
    b = (0.1 * rng.standard_normal(C)).astype(np.float32).astype(np.float64)
    dy = bf16(rng.standard_normal((M, C)))
    return x, g, b, dy


@pytest.mark.parametrize("M,C", LN_SHAPES)
def test_layernorm_forward(M, C):
    x, g, b, _ = _ln_inputs(M, C, M + C)
    y_ref, mean_ref, rstd_ref = ORC.layernorm_fwd(x, g, b)
    y = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(M, dtype=torch.float32, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    g2.gpt2k_layernorm_fwd(y, mean, rstd, dev(x), dev(g, torch.float32), dev(b, torch.float32), M, C)
    torch.cuda.synchronize()
    assert_close(host(y), y_ref, 2 ** -7, 2 ** -9 * rms(y_ref))
    assert_close(host(mean), mean_ref, 0.0, 1e-5 / rstd_ref)
    assert_close(host(rstd), rstd_ref, 1e-5, 0.0)


@pytest.mark.parametrize("M,C", LN_SHAPES)
@pytest.mark.parametrize("accumulate", [0, 1])
def test_layernorm_backward(M, C, accumulate):
    x, g, b, dy = _ln_inputs(M, C, 7 * M + C)
    rng = np.random.default_rng(M * C + accumulate)
    dx0 = bf16(rng.standard_normal((M, C))) if accumulate else np.zeros((M, C))
    dg0 = rng.standard_normal(C).astype(np.float32).astype(np.float64)
    db0 = rng.standard_normal(C).astype(np.float32).astype(np.float64)
    ds0 = rng.standard_normal(C).astype(np.float32).astype(np.float64)
    # the GPU's own statistics feed both sides (this isolates the backward)
    xd = dev(x)
    yd = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(M, dtype=torch.float32, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    gd = dev(g, torch.float32)
    g2.gpt2k_layernorm_fwd(yd, mean, rstd, xd, gd, dev(b, torch.float32), M, C)
    dx = dev(dx0)
    dg, db, ds = dev(dg0, torch.float32), dev(db0, torch.float32), dev(ds0, torch.float32)
    part = torch.empty(g2.gpt2k_layernorm_bwd_scratch(C), dtype=torch.float32, device="cuda")
    g2.gpt2k_layernorm_bwd(dx, dev(dy), xd, mean, rstd, gd, dg, db, ds, part, M, C, accumulate)
    torch.cuda.synchronize()
    m_h, r_h = host(mean), host(rstd)
    dx_ref, dg_ref, db_ref = ORC.layernorm_bwd(x, g, m_h, r_h, dy)
    dx_ref = dx_ref + dx0
    got = host(dx)
    assert_close(got, dx_ref, 2 ** -7, 2 ** -9 * rms(dx_ref))
    xh = (x - m_h[:, None]) * r_h[:, None]
    assert_close(host(dg), dg0 + dg_ref, 0.0, 1e-5 * np.abs(dy * xh).sum(axis=0) + 1e-6)
    assert_close(host(db), db0 + db_ref, 0.0, 1e-5 * np.abs(dy).sum(axis=0) + 1e-6)
    # dsum adds the column sums of dx exactly as stored
    assert_close(host(ds), ds0 + got.sum(axis=0), 0.0, 1e-5 * np.abs(got).sum(axis=0) + 1e-6)


def test_layernorm_backward_is_deterministic():
    M, C = 4096, 768
    x, g, b, dy = _ln_inputs(M, C, 3)
    xd, dyd, gd = dev(x), dev(dy), dev(g, torch.float32)
    y = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    mean = torch.empty(M, dtype=torch.float32, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    g2.gpt2k_layernorm_fwd(y, mean, rstd, xd, gd, dev(b, torch.float32), M, C)
    part = torch.empty(g2.gpt2k_layernorm_bwd_scratch(C), dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(2):
        dx = torch.zeros((M, C), dtype=torch.bfloat16, device="cuda")
        dg = torch.zeros(C, dtype=torch.float32, device="cuda")
        db = torch.zeros(C, dtype=torch.float32, device="cuda")
        ds = torch.zeros(C, dtype=torch.float32, device="cuda")
        g2.gpt2k_layernorm_bwd(dx, dyd, xd, mean, rstd, gd, dg, db, ds, part, M, C, 0)
        outs.append([t.cpu().view(torch.uint8).numpy().tobytes() for t in (dx, dg, db, ds)])
    assert outs[0] == outs[1]


def test_layernorm_rejects_bad_shapes():
    z = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(64, dtype=torch.float32, device="cuda")
    for C in (0, 12, 4096):
        with pytest.raises(g2.GPT2Error):
            g2.gpt2k_layernorm_fwd(z, f, f, z, f, f, 1, C)


# (M, V, Vp): padded and unpadded vocabularies; rows that fit the persistent
# shared-memory kernel twice (Vp <= 51200) and rows that do not (65536)
CLS_SHAPES = [(3, 8, 8), (4, 100, 104), (37, 1000, 1024), (300, 50257, 50304), (5, 65536, 65536)]


def _cls_inputs(M, V, Vp, seed):
    rng = np.random.default_rng(seed)
    z = bf16(3.0 * rng.standard_normal((M, Vp)))
    t = rng.integers(0, V, M).astype(np.int32)
    t[0] = 0
    t[-1] = V - 1
    return z, t


@pytest.mark.parametrize("M,V,Vp", CLS_SHAPES)
def test_classifier(M, V, Vp):
    z, t = _cls_inputs(M, V, Vp, M + V)
    losses_ref, dz_ref = ORC.softmax_xent(z[:, :V], t, 1.0)
    lse_ref = losses_ref + z[np.arange(M), t]
    zd = dev(z)
    losses = torch.empty(M, dtype=torch.float32, device="cuda")
    td = torch.tensor(t, device="cuda")
    g2.gpt2k_classifier(zd, losses, td, M, V, Vp, write_grad=True)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() == 0
    assert_close(host(losses), losses_ref, 0.0, 1e-5 * (1.0 + np.abs(lse_ref)))
    got = host(zd)
    assert_close(got[:, :V], dz_ref, 2 ** -7, 1e-3 * rms(dz_ref))
    assert np.all(got[:, V:] == 0.0)


def test_classifier_loss_only_leaves_logits():
    M, V, Vp = 64, 50257, 50304
    z, t = _cls_inputs(M, V, Vp, 11)
    losses_ref, _ = ORC.softmax_xent(z[:, :V], t, 1.0, grad=False)
    zd = dev(z)
    before = zd.clone()
    losses = torch.empty(M, dtype=torch.float32, device="cuda")
    g2.gpt2k_classifier(zd, losses, torch.tensor(t, device="cuda"), M, V, Vp, write_grad=False)
    torch.cuda.synchronize()
    assert torch.equal(zd, before)
    lse_ref = losses_ref + z[np.arange(M), t]
    assert_close(host(losses), losses_ref, 0.0, 1e-5 * (1.0 + np.abs(lse_ref)))


def test_classifier_bad_target_sets_error_bit():
    M, V, Vp = 4, 100, 104
    z, t = _cls_inputs(M, V, Vp, 5)
    t[1] = V  # out of range: read as class 0
    g2.gpt2k_take_error()
    zd = dev(z)
    losses = torch.empty(M, dtype=torch.float32, device="cuda")
    g2.gpt2k_classifier(zd, losses, torch.tensor(t, device="cuda"), M, V, Vp)
    torch.cuda.synchronize()
    assert g2.gpt2k_take_error() & 2
    t0 = t.copy()
    t0[1] = 0
    losses_ref, _ = ORC.softmax_xent(z[:, :V], t0, 1.0, grad=False)
    assert abs(float(losses[1]) - losses_ref[1]) < 1e-4 * (1 + abs(losses_ref[1]))
