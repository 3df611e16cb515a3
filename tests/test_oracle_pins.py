"""Pins for the CPU oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself -- a number
printed on the pages (tests/golden/page_numbers.json, each with its source),
a closed form, an invariant, a special case that reduces to a textbook
result, or brute force (central differences) on tiny shapes.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy import stats

import oracle
from oracle import Config, Oracle
from transformer_lm_pretraining_b200.inputs import iid_batch, ZipfStream

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_numbers.json")))


def closed_form_params(L, C, V, Tmax):
    return 12 * L * C * C + 13 * L * C + 2 * C + V * C + Tmax * C


# --------------------------------------------------------------- counts ----
def test_param_count_closed_form_and_pages():
    g = GOLDEN["gpt2_124m_param_count_closed_form"]
    s = g["shape"]
    o = Oracle(Config(s["L"], 12, s["C"], s["V"], s["V"], s["Tmax"]))
    assert o.num_params() == closed_form_params(s["L"], s["C"], s["V"], s["Tmax"]) == g["value"]

    ts = GOLDEN["param_count_tinystories"]
    s = ts["shape"]
    o = Oracle(Config(s["L"], s["H"], s["C"], s["V"], s["V"], s["Tmax"]))
    assert o.num_params() == ts["value"]
    sl = {n: num for n, _, num, _ in o.slices()}
    assert sl["wte"] + sl["wpe"] == ts["embeddings"]
    assert o.num_params() - sl["wte"] - sl["wpe"] == ts["non_embedding"]

    sm = GOLDEN["param_count_small_gpt"]
    s = sm["shape"]
    o = Oracle(Config(s["L"], s["H"], s["C"], s["V"], s["V"], s["Tmax"]))
    assert round(o.num_params() / 1e6, 2) == sm["value_rounded_millions"]

    tied = GOLDEN["gpt2_124m_tied_matrix"]
    n_tied = tied["vocab"] * tied["C"]
    assert round(n_tied / 1e6, 1) == tied["approx_params_millions"]
    assert round(100 * n_tied / 124e6) == tied["approx_share_percent"]


def test_padded_vocab_adds_only_pad_rows():
    a = Oracle(Config(12, 12, 768, 50257, 50257, 1024)).num_params()
    b = Oracle(Config(12, 12, 768, 50257, 50304, 1024)).num_params()
    assert b - a == (50304 - 50257) * 768
    assert b == 124475904


def test_decay_groups_are_the_2d_tensors():
    o = Oracle(Config(2, 2, 16, 11, 64, 5))
    dec = {n: d for n, _, _, d in o.slices()}
    assert {n for n, d in dec.items() if d} == {"wte", "wpe", "w_qkv", "w_o", "w_fc", "w_p"}


# ------------------------------------------------------------------ init ---
def test_splitmix64_reference_vectors():
    want = [int(x, 16) for x in GOLDEN["splitmix64_seed0"]["outputs"]]
    assert [oracle.splitmix64(0, n) for n in (1, 2, 3)] == want


def test_box_muller_is_standard_normal():
    z = np.array([oracle.std_normal(7, 4, i) for i in range(20000)])
    assert abs(z.mean()) < 4 / math.sqrt(z.size)
    assert abs(z.std() - 1) < 4 / math.sqrt(2 * z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_init_statistics_and_constants():
    cfg = Config(4, 4, 64, 300, 320, 32)
    o = Oracle(cfg)
    p = o.init(0)
    res_sd = 0.02 / math.sqrt(2 * cfg.L)
    for name, off, num, _ in o.slices():
        t = p[off:off + num]
        if name == "wte":
            real = t[: cfg.V * cfg.C]
            assert np.all(t[cfg.V * cfg.C:] == 0), "pad rows start at 0"
            t = real
        if name in ("wte", "wpe", "w_qkv", "w_fc", "w_o", "w_p"):
            sd = res_sd if name in ("w_o", "w_p") else 0.02
            n = t.size
            assert abs(t.mean()) < 5 * sd / math.sqrt(n), name
            assert abs(t.std() / sd - 1) < 5 / math.sqrt(2 * n), name
        elif name in ("ln1_g", "ln2_g", "lnf_g"):
            assert np.all(t == 1)
        else:
            assert np.all(t == 0), name
    # values are fp32-representable and seed-dependent
    assert np.all(p.astype(np.float32).astype(np.float64) == p)
    assert not np.array_equal(p, o.init(1))
    f = Oracle(cfg, np.float32).init(0)
    assert np.array_equal(f.astype(np.float64), p)


# ------------------------------------------------------------------ loss ---
def test_initial_loss_near_ln_v():
    for cfg, B, T in ((Config(2, 4, 128, 1024, 1024, 64), 4, 64),
                      (Config(2, 2, 64, 4096, 4096, 32), 2, 32)):
        o = Oracle(cfg)
        p = o.init(0)
        tok, tgt = iid_batch(cfg.V, B, T, seed=0)
        loss, losses, _ = o.forward(p, tok, tgt, B, T)
        assert abs(loss - math.log(cfg.V)) < 0.3
        # logits ~ N(0, C * 0.02^2): E[lse - z_tgt] ~ ln V + var / 2 where the
        # target is not the input token; with the tied matrix the input
        # token's own logit is large (~ rstd * |wte_tok|^2), so positions
        # whose target repeats the input token have a clearly lower loss.
        other = tok.ravel() != tgt.ravel()
        assert abs(losses[other].mean() - (math.log(cfg.V) + cfg.C * 0.02 ** 2 / 2)) < 0.05
        assert losses[~other].mean() < losses[other].mean() - 0.5


def test_page_initial_loss_is_near_ln_v_for_its_vocab():
    g = GOLDEN["initial_loss_tinystories"]
    assert abs(g["val_loss_step0"] - math.log(g["V"])) < 0.3


def test_uniform_special_case_closed_form():
    """wte = 0 => every logit is 0 => loss = ln V exactly and, with lnf_g = 0,
    lnf_b = beta, dwte[v] = beta * (1/V - count_v / M) * scale."""
    cfg = Config(2, 2, 16, 37, 64, 8)
    o = Oracle(cfg)
    p = o.init(3)
    o.view(p, "wte")[:] = 0
    o.view(p, "lnf_g")[:] = 0
    beta = np.linspace(-1, 1, cfg.C)
    o.view(p, "lnf_b")[:] = beta
    B, T = 3, 8
    tok, tgt = iid_batch(cfg.V, B, T, seed=5)
    loss, g, losses = o.forward_backward(p, tok, tgt, B, T, loss_scale=0.5)
    assert abs(loss - math.log(cfg.V)) < 1e-12
    assert np.allclose(losses, math.log(cfg.V), atol=1e-12, rtol=0)
    M = B * T
    counts = np.bincount(tgt.ravel(), minlength=cfg.Vp).astype(np.float64)
    want = 0.5 * np.outer(np.where(np.arange(cfg.Vp) < cfg.V, 1.0 / cfg.V, 0.0) - counts / M, beta)
    assert np.allclose(o.view(g, "wte").reshape(cfg.Vp, cfg.C), want, atol=1e-14, rtol=0)
    # nothing upstream of the (zero) head matrix receives gradient
    for name in ("wpe", "w_qkv", "w_fc", "w_o", "w_p", "lnf_g", "ln1_g"):
        assert np.all(o.view(g, name) == 0), name


# ------------------------------------------------------------- attention ---
def test_attention_single_position_returns_v():
    cfg = Config(1, 2, 16, 11, 11, 4)
    o = Oracle(cfg)
    rng = np.random.default_rng(0)
    qkv = rng.standard_normal((3, 3 * cfg.C))
    y = o.attention_fwd(qkv, B=3, T=1)
    assert np.array_equal(y, qkv[:, 2 * cfg.C:])


def test_attention_zero_query_is_causal_prefix_mean():
    cfg = Config(1, 2, 16, 11, 11, 9)
    o = Oracle(cfg)
    rng = np.random.default_rng(1)
    B, T = 2, 9
    qkv = rng.standard_normal((B * T, 3 * cfg.C))
    qkv[:, : cfg.C] = 0.0
    y = o.attention_fwd(qkv, B, T).reshape(B, T, cfg.C)
    v = qkv[:, 2 * cfg.C:].reshape(B, T, cfg.C)
    want = np.cumsum(v, axis=1) / np.arange(1, T + 1)[None, :, None]
    assert np.allclose(y, want, atol=1e-14)


def test_attention_is_causal_and_sharp_limit():
    cfg = Config(1, 1, 8, 11, 11, 6)
    o = Oracle(cfg)
    rng = np.random.default_rng(2)
    T = 6
    qkv = rng.standard_normal((T, 3 * cfg.C))
    y0 = o.attention_fwd(qkv, 1, T)
    qkv2 = qkv.copy()
    qkv2[4:, cfg.C:] += 10.0  # change keys/values of positions 4, 5
    y1 = o.attention_fwd(qkv2, 1, T)
    assert np.array_equal(y0[:4], y1[:4])
    assert not np.allclose(y0[4:], y1[4:])
    # a key aligned with the query and much larger than the rest wins
    qkv3 = np.zeros((T, 3 * cfg.C))
    qkv3[:, : cfg.C] = 1.0
    qkv3[2, cfg.C: 2 * cfg.C] = 50.0
    qkv3[:, 2 * cfg.C:] = rng.standard_normal((T, cfg.C))
    y = o.attention_fwd(qkv3, 1, T)
    assert np.allclose(y[2:], qkv3[2, 2 * cfg.C:], atol=1e-12)


# ------------------------------------------------------------- layernorm ---
def test_layernorm_output_moments():
    cfg = Config(1, 1, 32, 11, 11, 4)
    o = Oracle(cfg)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 32)) * 3 + 1
    y, mean, rstd = o.layernorm_fwd(x, np.ones(32), np.zeros(32))
    assert np.allclose(y.mean(1), 0, atol=1e-14)
    var = (x.var(1))
    assert np.allclose(rstd, 1 / np.sqrt(var + 1e-5), rtol=1e-14)
    assert np.allclose((y ** 2).mean(1), var / (var + 1e-5), rtol=1e-12)
    assert np.allclose(mean, x.mean(1), rtol=1e-14)


# ------------------------------------------------------------------ GELU ---
def test_layernorm_backward_matches_central_differences():
    # L = sum(w * LN(x)) for a fixed w: dL/dx, dL/dg, dL/db by central
    # differences of the forward against the backward with dy = w
    o = Oracle(Config(1, 1, 8, 11, 11, 4))
    rng = np.random.default_rng(5)
    M, C = 3, 8
    x = rng.standard_normal((M, C))
    g = 1.0 + 0.3 * rng.standard_normal(C)
    b = 0.1 * rng.standard_normal(C)
    w = rng.standard_normal((M, C))
    _, mean, rstd = o.layernorm_fwd(x, g, b)
    dx, dg, db = o.layernorm_bwd(x, g, mean, rstd, w)

    def loss(x_, g_, b_):
        return float((w * o.layernorm_fwd(x_, g_, b_)[0]).sum())

    h = 1e-6
    for arr, grad in ((x, dx), (g, dg), (b, db)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            e = np.zeros_like(arr)
            e[idx] = h
            args = [x, g, b]
            k = next(i for i, a in enumerate(args) if a is arr)
            args_p = list(args); args_p[k] = arr + e
            args_m = list(args); args_m[k] = arr - e
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.allclose(grad, num, rtol=1e-6, atol=1e-7)
    # shifting a row leaves LN unchanged: each row of dx sums to zero
    assert np.allclose(dx.sum(axis=1), 0.0, atol=1e-12)


def test_softmax_xent_closed_forms():
    o = Oracle(Config(1, 1, 8, 11, 11, 4))
    # uniform logits: loss = ln V, dz = (1/V - onehot) * scale / M exactly
    M, V, scale = 4, 7, 0.5
    z = np.full((M, V), 1.25)
    t = np.array([0, 3, 6, 2])
    losses, dz = o.softmax_xent(z, t, scale)
    assert np.allclose(losses, math.log(V), rtol=0, atol=1e-15)
    want = (np.full((M, V), 1.0 / V) - np.eye(V)[t]) * scale / M
    assert np.allclose(dz, want, rtol=0, atol=1e-16)
    # two classes: loss = softplus(z_other - z_target); rows of dz sum to 0
    rng = np.random.default_rng(6)
    z2 = rng.standard_normal((5, 2)) * 3
    t2 = rng.integers(0, 2, 5)
    l2, d2 = o.softmax_xent(z2, t2, 1.0)
    other = z2[np.arange(5), 1 - t2] - z2[np.arange(5), t2]
    assert np.allclose(l2, np.log1p(np.exp(other)), rtol=1e-14)
    assert np.allclose(d2.sum(axis=1), 0.0, atol=1e-16)
    # no gradient requested: losses only
    l3, d3 = o.softmax_xent(z2, t2, 1.0, grad=False)
    assert d3 is None and np.array_equal(l3, l2)


def test_gelu_identities():
    o = Oracle(Config(1, 1, 8, 11, 11, 4))
    xs = np.linspace(-8, 8, 321)
    gt = o.gelu_tanh(xs)
    ge = o.gelu_erf(xs)
    # 0.5 (1 + tanh(u)) = sigmoid(2u) with u = sqrt(2/pi)(x + 0.044715 x^3)
    u = math.sqrt(2 / math.pi) * (xs + 0.044715 * xs ** 3)
    assert np.allclose(gt, xs * stats.logistic.cdf(2 * u), rtol=1e-13, atol=1e-15)
    # exact GELU is x * Phi(x)
    assert np.allclose(ge, xs * stats.norm.cdf(xs), rtol=1e-12, atol=1e-15)
    assert o.gelu_tanh(0.0) == 0 and o.gelu_erf(0.0) == 0
    # GELU(x) - x/2 is even... i.e. x*(Phi(x) - 1/2) is even in x
    assert np.allclose(gt - xs / 2, (gt - xs / 2)[::-1], atol=1e-15)
    assert abs(o.gelu_tanh(8.0) - 8.0) < 1e-12 and abs(o.gelu_tanh(-8.0)) < 1e-12
    # the two forms differ (the page's logit mismatch) but by little
    d = np.abs(gt - ge)
    assert 1e-4 < d.max() < 1e-3
    # derivative against central differences
    h = 1e-6
    fd = (o.gelu_tanh(xs + h) - o.gelu_tanh(xs - h)) / (2 * h)
    assert np.allclose(o.gelu_tanh_grad(xs), fd, atol=1e-8)


# ------------------------------------------------------------- gradients ---
GRAD_SHAPES = [
    (Config(1, 1, 8, 11, 11, 5), 2, 1),
    (Config(1, 1, 8, 11, 64, 5), 2, 3),
    (Config(2, 2, 8, 11, 64, 5), 2, 5),
    (Config(1, 2, 16, 64, 128, 5), 2, 3),
    (Config(2, 2, 16, 64, 64, 5), 2, 5),
]


@pytest.mark.parametrize("cfg,B,T", GRAD_SHAPES)
def test_gradients_match_central_differences(cfg, B, T):
    o = Oracle(cfg)
    p = o.init(11)
    rng = np.random.default_rng(4)
    # move away from the symmetric init so every path carries gradient
    for name, off, num, _ in o.slices():
        p[off:off + num] += 0.05 * rng.standard_normal(num)
    p[o.slices()[0][1] + cfg.V * cfg.C: o.slices()[0][2]] = 0.0  # pad rows
    tok, tgt = iid_batch(cfg.V, B, T, seed=6)
    _, g, _ = o.forward_backward(p, tok, tgt, B, T, loss_scale=1.0)
    h = 1e-5
    fd = np.zeros_like(p)
    for i in range(p.size):
        old = p[i]
        p[i] = old + h
        lp = o.forward(p, tok, tgt, B, T)[0]
        p[i] = old - h
        lm = o.forward(p, tok, tgt, B, T)[0]
        p[i] = old
        fd[i] = (lp - lm) / (2 * h)
    for name, off, num, _ in o.slices():
        a, b = g[off:off + num], fd[off:off + num]
        scale = max(np.abs(b).max(), 1e-3)
        assert np.abs(a - b).max() <= 1e-6 * scale, (name, np.abs(a - b).max(), scale)
    # padded rows of wte never receive gradient
    assert np.all(o.view(g, "wte")[cfg.V * cfg.C:] == 0)


def test_padding_does_not_change_results():
    """Results with Vpad > V equal results with Vpad = V (pad rows are 0)."""
    a = Config(2, 2, 16, 37, 37, 8)
    b = Config(2, 2, 16, 37, 64, 8)
    oa, ob = Oracle(a), Oracle(b)
    pa = oa.init(9)
    pb = ob.init(9)
    B, T = 2, 8
    tok, tgt = iid_batch(a.V, B, T, seed=2)
    la, ga, _ = oa.forward_backward(pa, tok, tgt, B, T)
    lb, gb, _ = ob.forward_backward(pb, tok, tgt, B, T)
    assert la == lb
    for name, _, _, _ in oa.slices():
        x, y = oa.view(ga, name), ob.view(gb, name)
        if name == "wte":
            assert np.array_equal(x, y[: x.size]) and np.all(y[x.size:] == 0)
        else:
            assert np.array_equal(x, y), name
    assert np.array_equal(oa.view(pa, "wte"), ob.view(pb, "wte")[: a.V * a.C])


# ---------------------------------------------------------- accumulation ---
def test_micro_batch_accumulation_equals_full_batch():
    cfg = Config(2, 2, 16, 50, 64, 6)
    o = Oracle(cfg)
    p = o.init(1)
    n, Bm, T = 3, 2, 6
    s = ZipfStream(cfg.V, seed=0)
    chunks = [s.next_batch(Bm, T) for _ in range(n)]
    tok = np.concatenate([c[0] for c in chunks])
    tgt = np.concatenate([c[1] for c in chunks])
    full_loss, gfull, _ = o.forward_backward(p, tok, tgt, n * Bm, T, 1.0)
    acc = np.zeros_like(p)
    losses = []
    for t_, y_ in chunks:
        l, _, _ = o.forward_backward(p, t_, y_, Bm, T, 1.0 / n, acc)
        losses.append(l)
    assert abs(np.mean(losses) - full_loss) < 1e-12
    assert np.abs(acc - gfull).max() <= 1e-12 * np.abs(gfull).max()
    # without the 1/n scale the accumulated gradient is n times too large
    acc2 = np.zeros_like(p)
    for t_, y_ in chunks:
        o.forward_backward(p, t_, y_, Bm, T, 1.0, acc2)
    assert np.allclose(acc2, n * gfull, rtol=1e-10, atol=1e-15)


def test_stream_targets_are_tokens_shifted_by_one():
    s = ZipfStream(1000, seed=0)
    a_tok, a_tgt = s.next_batch(2, 8)
    b_tok, b_tgt = s.next_batch(2, 8)
    flat = np.concatenate([a_tok.ravel(), b_tok.ravel(), b_tgt.ravel()[-1:]])
    assert np.array_equal(a_tgt.ravel(), flat[1:17])
    assert np.array_equal(b_tgt.ravel(), flat[17:33])


# --------------------------------------------------------- clip / AdamW ---
def test_clip_properties():
    o = Oracle(Config(1, 1, 8, 11, 11, 4))
    rng = np.random.default_rng(5)
    g = rng.standard_normal(1000) * 0.3
    n0 = np.sqrt(np.sum(g.astype(np.longdouble) ** 2))
    gc = g.copy()
    n = o.clip(gc, 1.0)
    assert abs(n - float(n0)) < 1e-12 * float(n0)
    assert n > 1 and abs(np.linalg.norm(gc) - 1.0) < 1e-6
    small = g / (2 * float(n0))
    sc = small.copy()
    o.clip(sc, 1.0)
    assert np.array_equal(sc, small)


def test_adamw_first_two_steps_closed_form():
    cfg = Config(1, 1, 8, 11, 16, 4)
    o = Oracle(cfg)
    p0 = o.init(2)
    rng = np.random.default_rng(7)
    g = rng.standard_normal(p0.size)
    lr, wd, eps = 6e-4, 0.1, 1e-8
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    o.adamw(p, g, m, v, 1, lr, 0.9, 0.95, eps, wd)
    dec = np.zeros(p0.size, bool)
    for name, off, num, d in o.slices():
        dec[off:off + num] = d
    w = np.where(dec, wd, 0.0)
    want1 = p0 - lr * (g / (np.abs(g) + eps) + w * p0)
    assert np.allclose(p, want1, rtol=0, atol=1e-15)
    # same gradient again: bias-corrected moments are again g and g^2
    p1 = p.copy()
    o.adamw(p, g, m, v, 2, lr, 0.9, 0.95, eps, wd)
    want2 = p1 - lr * (g / (np.abs(g) + eps) + w * p1)
    assert np.allclose(p, want2, rtol=0, atol=1e-12)


def test_lr_schedule_endpoints():
    s = GOLDEN["gpt2_schedule"]
    W, S, mx = s["warmup"], s["max_steps"], s["max_lr"]
    mn = mx * s["min_lr_fraction"]
    assert oracle.lr(W - 1, mx, mn, W, S) == pytest.approx(mx, rel=1e-15)
    assert oracle.lr(0, mx, mn, W, S) == pytest.approx(mx / W, rel=1e-15)
    assert oracle.lr(S, mx, mn, W, S) == pytest.approx(mn, rel=1e-12)
    assert oracle.lr((W + S) // 2, mx, mn, W, S) == pytest.approx((mx + mn) / 2, rel=1e-6)
    assert oracle.lr(S + 10, mx, mn, W, S) == mn
    xs = [oracle.lr(k, mx, mn, W, S) for k in range(W, S + 1, 97)]
    assert all(a >= b for a, b in zip(xs, xs[1:]))
    assert s["tokens_per_step"] == 2 ** 19


def test_perplexity_and_bpb_identities():
    g = GOLDEN["perplexity"]
    assert round(math.exp(g["loss_nats"]), 2) == g["ppl"]
    assert round(g["loss_nats"] / math.log(2) / g["bpb"], 2) == g["bytes_per_token"]
    assert round(g["val_bytes"] / g["val_tokens"], 2) == g["bytes_per_token_check"]


# ---------------------------------------------------------- consistency ---
def test_openmp_build_is_bit_identical():
    cfg = Config(2, 2, 32, 100, 128, 16)
    a, b = Oracle(cfg), Oracle(cfg, openmp=True)
    p = a.init(0)
    tok, tgt = iid_batch(cfg.V, 2, 16, seed=1)
    la, ga, _ = a.forward_backward(p, tok, tgt, 2, 16)
    lb, gb, _ = b.forward_backward(p, tok, tgt, 2, 16)
    assert la == lb and np.array_equal(ga, gb)


def test_fp32_oracle_tracks_fp64():
    cfg = Config(2, 4, 64, 256, 256, 32)
    o64, o32 = Oracle(cfg), Oracle(cfg, np.float32)
    p = o64.init(0)
    tok, tgt = iid_batch(cfg.V, 2, 32, seed=0)
    l64, g64, _ = o64.forward_backward(p, tok, tgt, 2, 32)
    l32, g32, _ = o32.forward_backward(p.astype(np.float32), tok, tgt, 2, 32)
    assert abs(l64 - l32) < 1e-5
    for name, off, num, _ in o64.slices():
        a, b = g64[off:off + num], g32[off:off + num].astype(np.float64)
        if np.abs(a).max() == 0:
            continue
        assert np.abs(a - b).max() <= 1e-4 * np.abs(a).max(), name


def test_sample_token_is_the_inverse_cdf_of_the_tempered_softmax():
    o = Oracle(Config(1, 1, 8, 11, 11, 4))
    rng = np.random.default_rng(7)
    z = rng.standard_normal(9) * 2.0
    z[3] = z[6] = z.max() + 0.5  # a tie for the maximum
    # temperature 0: the argmax, the lowest index among equal maxima
    assert o.sample_token(z) == 3
    # a uniform grid of draws reproduces the softmax(z / T) masses exactly
    # (inverse-CDF construction), to within one grid step per token
    n = 20000
    for temp, k in ((1.0, 0), (0.7, 0), (2.0, 4)):
        counts = np.zeros(z.size)
        for i in range(n):
            counts[o.sample_token(z, temp, k, (i + 0.5) / n)] += 1
        keep = np.ones(z.size, bool)
        if k:
            keep = z >= np.sort(z)[::-1][k - 1]
        w = np.where(keep, np.exp((z - z.max()) / temp), 0.0)
        want = w / w.sum()
        assert np.all(np.abs(counts / n - want) <= 1.5 / n), (temp, k)
        assert np.all(counts[~keep] == 0)
    # a very low temperature concentrates on the (first) maximum
    assert all(o.sample_token(z, 1e-3, 0, u) in (3, 6) for u in (0.0, 0.3, 0.99))
