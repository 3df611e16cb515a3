"""Whole-step parity on the GPU: forward loss, every gradient tensor and the
post-AdamW parameters of the CUDA library against the CPU oracle (fp64) on
the same seeded inputs, for the fp32 validation build and the bf16 build;
plus determinism, bit-exact token handling, accumulation, checkpoint/resume
and the error paths.

Acceptance (the stated tolerances of the step):
  fp32 validation build: |loss - ref| <= 1e-4; per tensor max|g - ref| /
  max|ref| <= 1e-3 and cosine >= 0.99999.
  bf16 build: |loss - ref| <= 2e-2; per tensor cosine >= 0.995; parameters
  after one AdamW step within 2e-3 absolute.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import Config, Oracle
from transformer_lm_pretraining_b200.inputs import ZipfStream, iid_batch

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from transformer_lm_pretraining_b200 import gpt2 as g2  # noqa: E402

# (name, cfg, B, T): small enough for the oracle, several tiles + ragged tails
CASES = [
    ("tiny", Config(2, 4, 128, 1024, 1024, 64), 4, 64, True),      # the tiny single-step workload
    ("ragged", Config(2, 2, 128, 1000, 1024, 160), 2, 150, False),  # hd 64, ragged T and V
    ("hd128", Config(1, 2, 256, 777, 832, 96), 2, 96, False),       # hd 128, padded vocab
]


def tok_tensors(tok, tgt):
    return (torch.tensor(np.asarray(tok, np.int32), device="cuda"),
            torch.tensor(np.asarray(tgt, np.int32), device="cuda"))


def batch_for(cfg, B, T, iid, seed=0):
    if iid:
        return iid_batch(cfg.V, B, T, seed)
    return ZipfStream(cfg.V, seed).next_batch(B, T)


def per_tensor(o, a, b):
    out = {}
    for name, off, num, _ in o.slices():
        x, y = a[off:off + num].astype(np.float64), b[off:off + num].astype(np.float64)
        ny = np.abs(y).max()
        rel = np.abs(x - y).max() / ny if ny > 0 else np.abs(x).max()
        den = np.linalg.norm(x) * np.linalg.norm(y)
        cos = float(x @ y / den) if den > 0 else (1.0 if np.abs(x).max() == 0 else 0.0)
        out[name] = (rel, cos, ny)
    return out


def run_step(precision, cfg, B, T, tok, tgt, params, lr=6e-4):
    m = g2.GPT2(*cfg.args, seed=0, precision=precision, B=B, T=T)
    m.set_params(params.astype(np.float32))
    t, y = tok_tensors(tok, tgt)
    m.zero_grad()
    loss = m.forward(t, y)
    m.backward(1.0)
    grads = m.get_grads()
    norm = m.grad_norm_clip(1.0)
    m.adamw_step(lr, 0.9, 0.95, 1e-8, 0.1)
    post = m.get_params()
    losses = m.get_losses(B * T)
    m.close()
    return loss, grads, norm, post, losses


def oracle_step(cfg, B, T, tok, tgt, params, lr=6e-4):
    o = Oracle(cfg, openmp=True)
    p = params.astype(np.float64).copy()
    loss, g, losses = o.forward_backward(p, tok, tgt, B, T, 1.0)
    gc = g.copy()
    norm = o.clip(gc, 1.0)
    mm, vv = np.zeros_like(p), np.zeros_like(p)
    o.adamw(p, gc, mm, vv, 1, lr)
    return o, loss, g, norm, p, losses


@pytest.fixture(scope="module")
def oracle_runs():
    out = {}
    for name, cfg, B, T, iid in CASES:
        tok, tgt = batch_for(cfg, B, T, iid)
        params = Oracle(cfg).init(0).astype(np.float32)
        out[name] = (cfg, B, T, tok, tgt, params) + oracle_step(cfg, B, T, tok, tgt, params)
    return out


@pytest.mark.parametrize("case", [c[0] for c in CASES])
def test_fp32_build_matches_oracle(case, oracle_runs):
    cfg, B, T, tok, tgt, params, o, rloss, rg, rnorm, rpost, rlosses = oracle_runs[case]
    loss, g, norm, post, losses = run_step("fp32", cfg, B, T, tok, tgt, params)
    assert abs(loss - rloss) <= 1e-4
    assert np.abs(losses - rlosses).max() <= 1e-4
    for name, (rel, cos, ny) in per_tensor(o, g, rg).items():
        if ny == 0:
            assert rel == 0, name
            continue
        assert rel <= 1e-3 and cos >= 0.99999, (name, rel, cos)
    assert abs(norm - rnorm) <= 1e-4 * rnorm
    # One AdamW step moves p by lr * g / (|g| + eps) (+ decay): ~lr for every
    # element whose |g| >> eps, so an fp32-vs-fp64 difference in a gradient
    # near eps can move the update by up to 2 lr; elsewhere it agrees closely.
    d = np.abs(post - rpost)
    assert d.max() <= 2 * 6e-4
    assert np.mean(d > 1e-6) < 1e-3


@pytest.mark.parametrize("case", [c[0] for c in CASES])
def test_bf16_build_matches_oracle(case, oracle_runs):
    cfg, B, T, tok, tgt, params, o, rloss, rg, rnorm, rpost, rlosses = oracle_runs[case]
    loss, g, norm, post, losses = run_step("bf16", cfg, B, T, tok, tgt, params)
    assert abs(loss - rloss) <= 2e-2, (loss, rloss)
    for name, (rel, cos, ny) in per_tensor(o, g, rg).items():
        if ny == 0:
            assert rel == 0, name
            continue
        assert cos >= 0.995, (name, rel, cos)
    assert abs(norm - rnorm) <= 2e-2 * rnorm
    assert np.abs(post - rpost).max() <= 2e-3


def test_init_matches_oracle_init():
    cfg = Config(2, 4, 128, 1000, 1024, 64)
    m = g2.GPT2(*cfg.args, seed=1234, precision="bf16")
    got = m.get_params()
    m.close()
    want = Oracle(cfg).init(1234).astype(np.float32)
    # both round the same double to fp32; allow one fp32 ulp where libm differs
    ulp = np.spacing(np.abs(want).astype(np.float32))
    assert np.all(np.abs(got - want) <= ulp)
    assert np.mean(got == want) > 0.999


def test_token_handling_is_bit_exact():
    """wte row v encodes v and wpe row t encodes t with values exact in bf16;
    the layer-0 residual input must equal wte[tok] + wpe[t] exactly."""
    cfg = Config(1, 2, 128, 1000, 1024, 128)
    m = g2.GPT2(*cfg.args, seed=0, precision="bf16", B=2, T=128)
    o = Oracle(cfg)
    p = o.init(0).astype(np.float32)
    wte = o.view(p, "wte").reshape(cfg.Vp, cfg.C)
    wpe = o.view(p, "wpe").reshape(cfg.Tmax, cfg.C)
    v = np.arange(cfg.Vp, dtype=np.float32)
    wte[:] = 0
    wte[:, 0] = v           # integers < 256 are exact in bf16 ...
    wte[:, 1] = v % 256
    wte[:, 2] = np.floor(v / 256)
    wpe[:] = 0
    wpe[:, 3] = np.arange(cfg.Tmax)
    m.set_params(p)
    rng = np.random.default_rng(0)
    tok = rng.integers(0, cfg.V, size=(2, 128)).astype(np.int32)
    t, _ = tok_tensors(tok, tok)
    m.forward(t, None, sync_loss=False)
    x0 = m.read_activation("residual", 0, 2 * 128 * cfg.C).reshape(2, 128, cfg.C)
    m.close()
    flat = tok.reshape(2, 128)
    assert np.array_equal(x0[..., 1], flat % 256)
    assert np.array_equal(x0[..., 2], flat // 256)
    assert np.array_equal(x0[..., 3], np.broadcast_to(np.arange(128), (2, 128)))
    assert np.all(x0[..., 4:] == 0)


def test_bf16_runs_are_bit_identical():
    cfg = Config(2, 2, 128, 1000, 1024, 128)
    s = ZipfStream(cfg.V, 0)
    batches = [s.next_batch(2, 128) for _ in range(2)]
    res = []
    for _ in range(2):
        m = g2.GPT2(*cfg.args, seed=3, precision="bf16", B=2, T=128)
        losses = []
        for k, (tok, tgt) in enumerate(batches):
            t, y = tok_tensors(tok, tgt)
            m.zero_grad()
            losses.append(m.forward(t, y))
            m.backward(1.0)
            m.grad_norm_clip(1.0)
            m.adamw_step(1e-3)
        res.append((losses, m.get_params(), m.get_grads()))
        m.close()
    assert res[0][0] == res[1][0]
    assert np.array_equal(res[0][1], res[1][1])
    assert np.array_equal(res[0][2], res[1][2])


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_accumulation_equals_full_batch(precision):
    cfg = Config(2, 2, 128, 1000, 1024, 128)
    s = ZipfStream(cfg.V, 0)
    chunks = [s.next_batch(2, 128) for _ in range(2)]
    tok = np.concatenate([c[0] for c in chunks])
    tgt = np.concatenate([c[1] for c in chunks])
    m = g2.GPT2(*cfg.args, seed=5, precision=precision, B=4, T=128)
    t, y = tok_tensors(tok, tgt)
    m.zero_grad()
    full = m.forward(t, y)
    m.backward(1.0)
    gfull = m.get_grads()
    m.zero_grad()
    ls = []
    for a, b in chunks:
        ta, tb = tok_tensors(a, b)
        ls.append(m.forward(ta, tb))
        m.backward(0.5)
    gacc = m.get_grads()
    m.close()
    assert abs(np.mean(ls) - full) < (1e-5 if precision == "fp32" else 2e-3)
    cos = gacc @ gfull / (np.linalg.norm(gacc) * np.linalg.norm(gfull))
    assert cos > (0.999999 if precision == "fp32" else 0.999)
    assert abs(np.linalg.norm(gacc) / np.linalg.norm(gfull) - 1) < (1e-4 if precision == "fp32" else 1e-2)


def test_checkpoint_resume_is_bit_exact():
    cfg = Config(2, 2, 128, 1000, 1024, 128)
    s = ZipfStream(cfg.V, 0)
    batches = [tok_tensors(*s.next_batch(2, 128)) for _ in range(4)]

    def steps(m, bs, start):
        for k, (t, y) in enumerate(bs):
            m.zero_grad()
            m.forward(t, y, sync_loss=False)
            m.backward(1.0)
            m.grad_norm_clip(1.0, sync=False)
            m.adamw_step(g2.gpt2_lr(start + k, 1e-3, 1e-4, 2, 10))

    a = g2.GPT2(*cfg.args, seed=7, precision="bf16", B=2, T=128)
    steps(a, batches, 0)
    straight = a.get_params()
    a.close()
    b = g2.GPT2(*cfg.args, seed=7, precision="bf16", B=2, T=128)
    steps(b, batches[:2], 0)
    state = b.get_state()
    b.close()
    c = g2.GPT2(*cfg.args, seed=99, precision="bf16", B=2, T=128)
    c.set_state(*state)
    steps(c, batches[2:], 2)
    resumed = c.get_params()
    c.close()
    assert state[3] == 2
    assert np.array_equal(straight, resumed)


def test_error_paths():
    cfg = Config(1, 2, 128, 100, 128, 64)
    m = g2.GPT2(*cfg.args, seed=0, precision="bf16", B=1, T=64)
    with pytest.raises(g2.GPT2Error) as e:
        m.backward(1.0)
    assert e.value.code == -2
    tok = np.zeros((1, 64), np.int32)
    tok[0, 5] = cfg.V  # out of range: read as id 0 on the device, reported
    t, y = tok_tensors(tok, np.zeros((1, 64), np.int32))
    with pytest.raises(g2.GPT2Error) as e:
        m.forward(t, y)
    assert e.value.code == -3
    with pytest.raises(g2.GPT2Error) as e:
        m.forward(tok_tensors(np.zeros((1, 65), np.int32), np.zeros((1, 65), np.int32))[0], None)
    assert e.value.code == -1  # T > Tmax
    # a NaN parameter: non-finite loss is reported and AdamW leaves params alone
    p = m.get_params()
    p[0] = np.nan
    p2 = p.copy()
    m.set_params(p)
    t, y = tok_tensors(np.zeros((1, 64), np.int32), np.zeros((1, 64), np.int32))
    with pytest.raises(g2.GPT2Error) as e:
        m.forward(t, y)
    assert e.value.code == -4
    m.backward(1.0)
    with pytest.raises(g2.GPT2Error) as e:
        m.grad_norm_clip(1.0)
    assert e.value.code == -4
    m.adamw_step(1e-3)
    after = m.get_params()
    assert np.array_equal(np.isnan(after), np.isnan(p2))
    assert np.array_equal(after[1:], p2[1:])
    m.close()


def test_clip_scale_matches_oracle_and_applies_once():
    cfg = Config(1, 2, 128, 500, 512, 64)
    o = Oracle(cfg)
    p = o.init(0)
    tok, tgt = ZipfStream(cfg.V, 0).next_batch(2, 64)
    _, g, _ = o.forward_backward(p, tok, tgt, 2, 64, 1.0)
    n_ref = o.grad_norm(g)
    m = g2.GPT2(*cfg.args, seed=0, precision="fp32", B=2, T=64)
    t, y = tok_tensors(tok, tgt)
    m.zero_grad()
    m.forward(t, y)
    m.backward(1.0)
    max_norm = n_ref / 4
    n = m.grad_norm_clip(max_norm)
    assert abs(n - n_ref) <= 1e-4 * n_ref
    p0, m0, v0, _ = m.get_state()
    m.adamw_step(1e-3, wd=0.0)
    _, m1, v1, t1 = m.get_state()
    gscaled = m.get_grads() * (max_norm / (n + 1e-6))
    assert np.allclose(m1, 0.1 * gscaled, rtol=1e-5, atol=1e-12)
    # the next step without a new clip uses scale 1
    m.adamw_step(1e-3, wd=0.0)
    _, m2, _, t2 = m.get_state()
    assert t2 == t1 + 1
    assert np.allclose(m2, 0.9 * m1 + 0.1 * m.get_grads(), rtol=1e-5, atol=1e-12)
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_evaluate_matches_oracle_forward(precision):
    # forward-only evaluation: the loss of the oracle's forward, the same
    # per-position losses as the training forward, logits left as computed,
    # no backward after it, and no effect on a training step that follows
    name, cfg, B, T, iid = CASES[1]
    tok, tgt = batch_for(cfg, B, T, iid, seed=3)
    params = Oracle(cfg).init(0).astype(np.float32)
    rloss, rlosses, _ = Oracle(cfg, openmp=True).forward(params.astype(np.float64), tok, tgt, B, T)
    m = g2.GPT2(*cfg.args, seed=0, precision=precision, B=B, T=T)
    m.set_params(params)
    t, y = tok_tensors(tok, tgt)
    loss = m.evaluate(t, y)
    tol = 1e-4 if precision == "fp32" else 2e-2
    assert abs(loss - rloss) <= tol, (loss, rloss)
    assert abs(math.exp(loss) - math.exp(rloss)) <= 2 * tol * math.exp(rloss)  # perplexity
    eval_losses = m.get_losses(B * T)
    eval_logits = m.logits(B, T).clone()
    with pytest.raises(g2.GPT2Error):
        m.backward(1.0)
    m.forward(t)  # no targets: logits only
    assert torch.equal(m.logits(B, T), eval_logits)
    # the training forward gives the same losses bit for bit; a step after
    # an evaluation equals a step without one
    m.zero_grad()
    assert m.forward(t, y) == loss
    assert np.array_equal(m.get_losses(B * T), eval_losses)
    m.backward(1.0)
    g_after = m.get_grads()
    m.close()
    m2 = g2.GPT2(*cfg.args, seed=0, precision=precision, B=B, T=T)
    m2.set_params(params)
    m2.zero_grad()
    m2.forward(t, y)
    m2.backward(1.0)
    assert np.array_equal(m2.get_grads(), g_after)
    m2.close()


def test_evaluate_at_a_smaller_batch_than_reserved():
    name, cfg, B, T, iid = CASES[0]
    tok, tgt = batch_for(cfg, B, T, iid, seed=4)
    params = Oracle(cfg).init(0).astype(np.float32)
    m = g2.GPT2(*cfg.args, seed=0, precision="bf16", B=B, T=T)
    m.set_params(params)
    t, y = tok_tensors(tok[:1, : T // 2], tgt[:1, : T // 2])
    loss = m.evaluate(t.contiguous(), y.contiguous())
    rloss, _, _ = Oracle(cfg).forward(params.astype(np.float64), tok[:1, : T // 2], tgt[:1, : T // 2],
                                      1, T // 2)
    assert abs(loss - rloss) <= 2e-2
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_recompute_is_bit_identical(precision):
    # GELU recomputed in the backward from the stored pre-activation gives
    # the same loss, gradients and updated parameters bit for bit, in a
    # workspace smaller by (L - 1) B T 4C activations
    name, cfg, B, T, iid = CASES[1]
    tok, tgt = batch_for(cfg, B, T, iid, seed=5)
    params = Oracle(cfg).init(0).astype(np.float32)
    out = []
    for level in (0, 1):
        m = g2.GPT2(*cfg.args, seed=0, precision=precision, B=B, T=T, recompute=level)
        m.set_params(params)
        t, y = tok_tensors(tok, tgt)
        m.zero_grad()
        loss = m.forward(t, y)
        m.backward(1.0)
        grads = m.get_grads()
        m.grad_norm_clip(1.0)
        m.adamw_step(6e-4, 0.9, 0.95, 1e-8, 0.1)
        out.append((loss, grads, m.get_params(), m.workspace_bytes(B, T)))
        if level:
            with pytest.raises(g2.GPT2Error):
                m.read_activation("gelu", 0, B * T * 4 * cfg.C)
        m.close()
    (l0, g0, p0, w0), (l1, g1, p1, w1) = out
    assert l0 == l1
    assert np.array_equal(g0, g1)
    assert np.array_equal(p0, p1)
    elt = 4 if precision == "fp32" else 2
    saved = (cfg.L - 1) * B * T * 4 * cfg.C * elt
    assert saved - 1024 <= w0 - w1 <= saved + 1024


def test_captured_step_equals_eager_steps():
    """The step captured as one CUDA graph (gpt2_step_graph_capture: zero
    grad, two micro-batches at loss scale 1/2, clip, AdamW with the schedule
    on the device) replays bit-identically to the same eager calls with the
    host's gpt2_lr, through the warmup and into the cosine phase."""
    cfg = Config(2, 2, 128, 1000, 1024, 128)
    B, T, n_micro = 2, 128, 2
    sched = (1e-3, 1e-4, 3, 10)  # steps 0-2 warm up, step 3 starts the cosine
    s = ZipfStream(cfg.V, 0)
    steps = [[s.next_batch(B, T) for _ in range(n_micro)] for _ in range(4)]
    stream = torch.cuda.Stream()

    def eager(m, k):
        m.zero_grad()
        for tok, tgt in steps[k]:
            t, y = tok_tensors(tok, tgt)
            m.forward(t, y, sync_loss=False)
            m.backward(1.0 / n_micro)
        m.grad_norm_clip(1.0, sync=False)
        m.adamw_step(g2.gpt2_lr(k, *sched), 0.9, 0.95, 1e-8, 0.1)
        return m.read_loss()

    with torch.cuda.stream(stream):
        a = g2.GPT2(*cfg.args, seed=7, precision="bf16", B=B, T=T)
        a.set_stream(stream)
        want = [eager(a, k) for k in range(4)]
        pa, ma, va, ta = a.get_state()
        a.close()

        b = g2.GPT2(*cfg.args, seed=7, precision="bf16", B=B, T=T)
        b.set_stream(stream)
        got = [eager(b, 0)]  # one eager step first: kernels set up outside the capture
        stok = torch.empty(n_micro * B * T, dtype=torch.int32, device="cuda")
        stgt = torch.empty(n_micro * B * T, dtype=torch.int32, device="cuda")
        kernels = b.capture_step(stok, stgt, B, T, n_micro, 1.0, *sched)
        assert kernels > 10
        for k in range(1, 4):
            for j, (tok, tgt) in enumerate(steps[k]):
                t, y = tok_tensors(tok, tgt)
                stok[j * B * T:(j + 1) * B * T].copy_(t.view(-1))
                stgt[j * B * T:(j + 1) * B * T].copy_(y.view(-1))
            b.launch_step()
            got.append(b.read_loss())
        pb, mb, vb, tb = b.get_state()
        b.close()
    assert got == want
    assert ta == tb == 4
    assert np.array_equal(pa, pb) and np.array_equal(ma, mb) and np.array_equal(va, vb)


def test_programmatic_launch_leaves_the_step_unchanged():
    """Kernels launched with programmatic stream serialization (each waits
    for its predecessors before touching global memory) give the same bits
    as plain launches: two eager steps and two graph replays of a step with
    a sequence of 1024 (several attention tiles, split-K weight gradients)."""
    cfg = Config(2, 2, 128, 1000, 1024, 1024)
    B, T = 2, 1024
    s = ZipfStream(cfg.V, 5)
    steps = [[s.next_batch(B, T)] for _ in range(4)]
    stream = torch.cuda.Stream()

    def run(pdl):
        prev = g2.gpt2k_set_programmatic_launch(pdl)
        try:
            with torch.cuda.stream(stream):
                m = g2.GPT2(*cfg.args, seed=11, precision="bf16", B=B, T=T)
                m.set_stream(stream)
                losses = []
                for k in range(2):
                    (tok, tgt), = steps[k]
                    t, y = tok_tensors(tok, tgt)
                    m.zero_grad()
                    m.forward(t, y, sync_loss=False)
                    m.backward(1.0)
                    m.grad_norm_clip(1.0, sync=False)
                    m.adamw_step(g2.gpt2_lr(k, 1e-3, 1e-4, 2, 10), 0.9, 0.95, 1e-8, 0.1)
                    losses.append(m.read_loss())
                stok = torch.empty(B * T, dtype=torch.int32, device="cuda")
                stgt = torch.empty(B * T, dtype=torch.int32, device="cuda")
                m.capture_step(stok, stgt, B, T, 1, 1.0, 1e-3, 1e-4, 2, 10)
                for k in range(2, 4):
                    (tok, tgt), = steps[k]
                    t, y = tok_tensors(tok, tgt)
                    stok.copy_(t.view(-1))
                    stgt.copy_(y.view(-1))
                    m.launch_step()
                    losses.append(m.read_loss())
                state = m.get_state()
                grads = m.get_grads()
                m.close()
        finally:
            g2.gpt2k_set_programmatic_launch(prev)
        return losses, state, grads

    off, on = run(0), run(1)
    assert off[0] == on[0]
    for a, b in zip(off[1][:3], on[1][:3]):
        assert np.array_equal(a, b)
    assert np.array_equal(off[2], on[2])
