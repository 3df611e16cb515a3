"""CPU oracle for one GPT-2 pretraining step.

TEST INFRASTRUCTURE ONLY.  The oracle is a plain, slow, single-threaded C++
statement of the step (``gpt2_oracle.cpp``), loaded here through ctypes.  Only
the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The CUDA library never calls it and the two share no
code: the only module both sides use is the seeded input generator
(``transformer_lm_pretraining_b200.inputs``), which holds none of the
method's arithmetic.

``build()`` compiles two variants: the plain single-threaded library and a
``-fopenmp`` build whose loops run in parallel only over independent output
elements (so its results are bit-identical to the single-threaded build).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gpt2_oracle.cpp")
_OUT = os.path.join(_HERE, "_build")

_LIBS: dict = {}


def _lib_path(openmp: bool) -> str:
    return os.path.join(_OUT, "liboracle_omp.so" if openmp else "liboracle.so")


def build(openmp: bool | None = None, force: bool = False) -> None:
    """Compile the oracle (both variants unless ``openmp`` is given)."""
    os.makedirs(_OUT, exist_ok=True)
    variants = [False, True] if openmp is None else [openmp]
    for omp in variants:
        out = _lib_path(omp)
        if (not force and os.path.exists(out)
                and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
            continue
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-o", out + ".tmp", _SRC]
        if omp:
            cmd.insert(1, "-fopenmp")
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)


_F64 = ctypes.POINTER(ctypes.c_double)
_F32 = ctypes.POINTER(ctypes.c_float)
_I32 = ctypes.POINTER(ctypes.c_int)


def lib(openmp: bool = False) -> ctypes.CDLL:
    if openmp in _LIBS:
        return _LIBS[openmp]
    build(openmp)
    L = ctypes.CDLL(_lib_path(openmp))
    sz, i, d, f, u64, lng = (ctypes.c_size_t, ctypes.c_int, ctypes.c_double,
                             ctypes.c_float, ctypes.c_uint64, ctypes.c_long)
    L.orc_num_params.argtypes = [i, i, i, i, i]
    L.orc_num_params.restype = sz
    L.orc_tensor_slice.argtypes = [i, i, i, i, i, i, ctypes.POINTER(sz),
                                   ctypes.POINTER(sz), ctypes.POINTER(i)]
    L.orc_tensor_slice.restype = i
    L.orc_std_normal.argtypes = [u64, i, u64]
    L.orc_std_normal.restype = d
    L.orc_splitmix64.argtypes = [u64, u64]
    L.orc_splitmix64.restype = u64
    L.orc_lr.argtypes = [lng, d, d, lng, lng]
    L.orc_lr.restype = d
    L.orc_openmp_threads.argtypes = []
    L.orc_openmp_threads.restype = i
    for sfx, R, P in (("f64", d, _F64), ("f32", f, _F32)):
        fn = getattr(L, f"orc_init_{sfx}")
        fn.argtypes = [i, i, i, i, i, i, u64, P]
        fn.restype = None
        fn = getattr(L, f"orc_forward_{sfx}")
        fn.argtypes = [i, i, i, i, i, i, P, _I32, _I32, i, i, P, P]
        fn.restype = R
        fn = getattr(L, f"orc_forward_backward_{sfx}")
        fn.argtypes = [i, i, i, i, i, i, P, _I32, _I32, i, i, R, P, P]
        fn.restype = R
        fn = getattr(L, f"orc_grad_norm_{sfx}")
        fn.argtypes = [P, sz]
        fn.restype = R
        fn = getattr(L, f"orc_clip_{sfx}")
        fn.argtypes = [P, sz, R]
        fn.restype = R
        fn = getattr(L, f"orc_adamw_{sfx}")
        fn.argtypes = [i, i, i, i, i, P, P, P, P, lng, R, R, R, R, R]
        fn.restype = None
        for name in ("gelu_tanh", "gelu_tanh_grad", "gelu_erf"):
            fn = getattr(L, f"orc_{name}_{sfx}")
            fn.argtypes = [R]
            fn.restype = R
        fn = getattr(L, f"orc_gelu_tanh_vec_{sfx}")
        fn.argtypes = [P, P, sz, i]
        fn.restype = None
        fn = getattr(L, f"orc_layernorm_fwd_{sfx}")
        fn.argtypes = [P, P, P, P, P, P, i, i]
        fn.restype = None
        fn = getattr(L, f"orc_layernorm_bwd_{sfx}")
        fn.argtypes = [P, P, P, P, P, P, P, P, i, i]
        fn.restype = None
        fn = getattr(L, f"orc_softmax_xent_{sfx}")
        fn.argtypes = [P, i, i, _I32, R, P, P]
        fn.restype = None
        fn = getattr(L, f"orc_sample_token_{sfx}")
        fn.argtypes = [P, i, R, i, d]
        fn.restype = i
        fn = getattr(L, f"orc_attention_fwd_{sfx}")
        fn.argtypes = [P, P, i, i, i, i]
        fn.restype = None
        fn = getattr(L, f"orc_attention_bwd_{sfx}")
        fn.argtypes = [P, P, P, i, i, i, i]
        fn.restype = None
        fn = getattr(L, f"orc_linear_fwd_{sfx}")
        fn.argtypes = [P, P, P, P, i, i, i]
        fn.restype = None
    _LIBS[openmp] = L
    return L


TENSOR_NAMES = ("wte", "wpe", "ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
                "ln2_g", "ln2_b", "w_fc", "b_fc", "w_p", "b_p", "lnf_g", "lnf_b")


@dataclass(frozen=True)
class Config:
    L: int
    H: int
    C: int
    V: int
    Vp: int
    Tmax: int

    @property
    def args(self):
        return (self.L, self.H, self.C, self.V, self.Vp, self.Tmax)


def _ptr(a: np.ndarray, dt):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(dt))


def _sfx(dtype):
    dtype = np.dtype(dtype)
    if dtype == np.float64:
        return "f64", ctypes.c_double
    if dtype == np.float32:
        return "f32", ctypes.c_float
    raise TypeError(dtype)


class Oracle:
    """Thin numpy-facing wrapper of the C oracle for one model shape."""

    def __init__(self, cfg: Config, dtype=np.float64, openmp: bool = False):
        self.cfg = cfg
        self.dtype = np.dtype(dtype)
        self.sfx, self.ct = _sfx(self.dtype)
        self.lib = lib(openmp)

    # layout -------------------------------------------------------------
    def num_params(self) -> int:
        c = self.cfg
        return int(self.lib.orc_num_params(c.L, c.C, c.V, c.Vp, c.Tmax))

    def slices(self):
        """[(name, offset, numel, decayed)] in flat order."""
        c = self.cfg
        out = []
        for i, name in enumerate(TENSOR_NAMES):
            off, num, dec = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int()
            rc = self.lib.orc_tensor_slice(c.L, c.C, c.V, c.Vp, c.Tmax, i,
                                           ctypes.byref(off), ctypes.byref(num),
                                           ctypes.byref(dec))
            assert rc == 0
            out.append((name, off.value, num.value, bool(dec.value)))
        return out

    def view(self, flat: np.ndarray, name: str) -> np.ndarray:
        for n, off, num, _ in self.slices():
            if n == name:
                return flat[off:off + num]
        raise KeyError(name)

    # step pieces --------------------------------------------------------
    def init(self, seed: int) -> np.ndarray:
        p = np.zeros(self.num_params(), self.dtype)
        getattr(self.lib, f"orc_init_{self.sfx}")(*self.cfg.args, seed, _ptr(p, self.ct))
        return p

    def forward(self, params, tok, tgt=None, B=None, T=None, want_logits=False):
        tok = np.ascontiguousarray(tok, np.int32).reshape(-1)
        B = B if B is not None else 1
        T = T if T is not None else tok.size // B
        M = B * T
        losses = np.zeros(M, self.dtype)
        logits = np.zeros((M, self.cfg.V), self.dtype) if want_logits else None
        tg = None if tgt is None else np.ascontiguousarray(tgt, np.int32).reshape(-1)
        p = np.ascontiguousarray(params, self.dtype)
        loss = getattr(self.lib, f"orc_forward_{self.sfx}")(
            *self.cfg.args, _ptr(p, self.ct), _ptr(tok, ctypes.c_int),
            None if tg is None else _ptr(tg, ctypes.c_int), B, T,
            _ptr(losses, self.ct) if tg is not None else None,
            _ptr(logits, self.ct) if want_logits else None)
        return float(loss), (losses if tg is not None else None), logits

    def forward_backward(self, params, tok, tgt, B, T, loss_scale=1.0, grads=None):
        """Returns (mean loss, grads += d(loss_scale * loss)/dparams, losses)."""
        tok = np.ascontiguousarray(tok, np.int32).reshape(-1)
        tgt = np.ascontiguousarray(tgt, np.int32).reshape(-1)
        p = np.ascontiguousarray(params, self.dtype)
        if grads is None:
            grads = np.zeros(self.num_params(), self.dtype)
        losses = np.zeros(B * T, self.dtype)
        loss = getattr(self.lib, f"orc_forward_backward_{self.sfx}")(
            *self.cfg.args, _ptr(p, self.ct), _ptr(tok, ctypes.c_int),
            _ptr(tgt, ctypes.c_int), B, T, loss_scale, _ptr(grads, self.ct),
            _ptr(losses, self.ct))
        return float(loss), grads, losses

    def grad_norm(self, grads) -> float:
        return float(getattr(self.lib, f"orc_grad_norm_{self.sfx}")(_ptr(grads, self.ct), grads.size))

    def clip(self, grads, max_norm=1.0) -> float:
        return float(getattr(self.lib, f"orc_clip_{self.sfx}")(_ptr(grads, self.ct), grads.size, max_norm))

    def adamw(self, params, grads, m, v, t, lr, b1=0.9, b2=0.95, eps=1e-8, wd=0.1):
        c = self.cfg
        getattr(self.lib, f"orc_adamw_{self.sfx}")(
            c.L, c.C, c.V, c.Vp, c.Tmax, _ptr(params, self.ct), _ptr(grads, self.ct),
            _ptr(m, self.ct), _ptr(v, self.ct), t, lr, b1, b2, eps, wd)

    # primitives ---------------------------------------------------------
    def _gelu_vec(self, x, grad):
        x = np.ascontiguousarray(x, self.dtype)
        y = np.empty_like(x)
        getattr(self.lib, f"orc_gelu_tanh_vec_{self.sfx}")(_ptr(x, self.ct), _ptr(y, self.ct),
                                                           x.size, int(grad))
        return y

    def gelu_tanh(self, x):
        if np.ndim(x) == 0:
            return float(getattr(self.lib, f"orc_gelu_tanh_{self.sfx}")(float(x)))
        return self._gelu_vec(x, False)

    def gelu_tanh_grad(self, x):
        if np.ndim(x) == 0:
            return float(getattr(self.lib, f"orc_gelu_tanh_grad_{self.sfx}")(float(x)))
        return self._gelu_vec(x, True)

    def gelu_erf(self, x):
        f = getattr(self.lib, f"orc_gelu_erf_{self.sfx}")
        return np.array([f(float(v)) for v in np.ravel(x)], self.dtype).reshape(np.shape(x))

    def attention_fwd(self, qkv, B, T):
        c = self.cfg
        qkv = np.ascontiguousarray(qkv, self.dtype)
        y = np.zeros((B * T, c.C), self.dtype)
        getattr(self.lib, f"orc_attention_fwd_{self.sfx}")(_ptr(qkv, self.ct), _ptr(y, self.ct), B, T, c.C, c.H)
        return y

    def attention_bwd(self, qkv, dy, B, T):
        c = self.cfg
        qkv = np.ascontiguousarray(qkv, self.dtype)
        dy = np.ascontiguousarray(dy, self.dtype)
        dqkv = np.zeros((B * T, 3 * c.C), self.dtype)
        getattr(self.lib, f"orc_attention_bwd_{self.sfx}")(_ptr(qkv, self.ct), _ptr(dy, self.ct),
                                                           _ptr(dqkv, self.ct), B, T, c.C, c.H)
        return dqkv

    def layernorm_fwd(self, x, g, b):
        x = np.ascontiguousarray(x, self.dtype)
        M, C = x.shape
        y = np.zeros_like(x)
        mean = np.zeros(M, self.dtype)
        rstd = np.zeros(M, self.dtype)
        getattr(self.lib, f"orc_layernorm_fwd_{self.sfx}")(
            _ptr(x, self.ct), _ptr(np.ascontiguousarray(g, self.dtype), self.ct),
            _ptr(np.ascontiguousarray(b, self.dtype), self.ct), _ptr(y, self.ct),
            _ptr(mean, self.ct), _ptr(rstd, self.ct), M, C)
        return y, mean, rstd

    def layernorm_bwd(self, x, g, mean, rstd, dy):
        """(dx, dg, db) of the LayerNorm backward (dx from zero)."""
        x = np.ascontiguousarray(x, self.dtype)
        M, C = x.shape
        dx = np.zeros_like(x)
        dg = np.zeros(C, self.dtype)
        db = np.zeros(C, self.dtype)
        getattr(self.lib, f"orc_layernorm_bwd_{self.sfx}")(
            _ptr(x, self.ct), _ptr(np.ascontiguousarray(g, self.dtype), self.ct),
            _ptr(np.ascontiguousarray(mean, self.dtype), self.ct),
            _ptr(np.ascontiguousarray(rstd, self.dtype), self.ct),
            _ptr(np.ascontiguousarray(dy, self.dtype), self.ct), _ptr(dx, self.ct),
            _ptr(dg, self.ct), _ptr(db, self.ct), M, C)
        return dx, dg, db

    def softmax_xent(self, z, tgt, scale=1.0, grad=True):
        """(losses, dz) of softmax cross-entropy over rows of z [M, V]; dz =
        (softmax - onehot) * scale / M, or None when grad is False."""
        z = np.ascontiguousarray(z, self.dtype)
        M, V = z.shape
        t = np.ascontiguousarray(tgt, np.int32)
        losses = np.zeros(M, self.dtype)
        dz = np.zeros_like(z) if grad else None
        getattr(self.lib, f"orc_softmax_xent_{self.sfx}")(
            _ptr(z, self.ct), M, V, t.ctypes.data_as(_I32),
            self.ct(scale), _ptr(losses, self.ct), _ptr(dz, self.ct) if grad else None)
        return losses, dz

    def sample_token(self, z, temperature=0.0, top_k=0, u=0.0):
        """Next token from one row of logits: argmax at temperature 0, else
        the first index where the cumulative softmax(z / temperature) over
        the top_k logits exceeds u."""
        z = np.ascontiguousarray(z, self.dtype)
        return int(getattr(self.lib, f"orc_sample_token_{self.sfx}")(
            _ptr(z, self.ct), z.size, self.ct(temperature), int(top_k), float(u)))

    def linear_fwd(self, x, W, b=None):
        x = np.ascontiguousarray(x, self.dtype)
        W = np.ascontiguousarray(W, self.dtype)
        M, K = x.shape
        N = W.shape[0]
        y = np.zeros((M, N), self.dtype)
        bb = None if b is None else _ptr(np.ascontiguousarray(b, self.dtype), self.ct)
        getattr(self.lib, f"orc_linear_fwd_{self.sfx}")(_ptr(x, self.ct), _ptr(W, self.ct), bb,
                                                        _ptr(y, self.ct), M, K, N)
        return y


def lr(step, max_lr, min_lr, warmup, max_steps) -> float:
    return float(lib().orc_lr(step, max_lr, min_lr, warmup, max_steps))


def splitmix64(seed: int, n: int) -> int:
    return int(lib().orc_splitmix64(seed, n))


def sample_uniform(seed: int, position: int, row: int) -> float:
    """The uniform draw for the token at `position` of sequence `row`:
    the SplitMix64 output n = position * 65536 + row of `seed`, top 53 bits."""
    return (splitmix64(seed, position * 65536 + row) >> 11) * 2.0 ** -53


def std_normal(seed: int, tensor: int, i: int) -> float:
    return float(lib().orc_std_normal(seed, tensor, i))


def openmp_threads() -> int:
    return int(lib(True).orc_openmp_threads())
