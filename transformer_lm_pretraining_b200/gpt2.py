"""ctypes binding of the GPT-2 step library (include/gpt2.h, gpt2_kernels.h).

Argument marshalling only: every step of the path runs in the CUDA library.
PyTorch provides device memory and the current stream.  The module-level
functions carry the C names; ``GPT2`` bundles them for one model.

The library is loaded from this package's ``lib/`` folder (built in-tree by
``python -m transformer_lm_pretraining_b200.build``).  A missing library is
an error: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIBDIR = os.path.join(HERE, "lib")

ERRORS = {-1: "GPT2_ERR_ARG", -2: "GPT2_ERR_STATE", -3: "GPT2_ERR_TOKEN",
          -4: "GPT2_ERR_NONFINITE", -5: "GPT2_ERR_CUDA", -6: "GPT2_ERR_TIMEOUT"}

ACT_NAMES = {"residual": 0, "ln1": 1, "qkv": 2, "attn": 3, "xmid": 4, "ln2": 5,
             "fc_pre": 6, "gelu": 7, "lnf": 8}

EPI = {"store": 0, "bias": 1, "bias_gelu": 2, "bias_resid": 3, "dgelu": 4, "f32_acc": 5}

PROF_KINDS = ("gemm", "attn_fwd", "attn_bwd", "ln_fwd", "ln_bwd", "classifier", "encoder",
              "colsum", "optimizer", "recompute")

# name -> (restype, argtypes)
_vp, _sz, _i, _f, _d, _l, _u64 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float,
                                  ctypes.c_double, ctypes.c_long, ctypes.c_uint64)
_fp = ctypes.POINTER(ctypes.c_float)
SIGNATURES = {
    "gpt2_build_is_bf16": (_i, []),
    "gpt2_create": (_i, [_i, _i, _i, _i, _i, _i, _u64, ctypes.POINTER(_vp)]),
    "gpt2_destroy": (None, [_vp]),
    "gpt2_num_params": (_sz, [_vp]),
    "gpt2_state_bytes": (_sz, [_vp]),
    "gpt2_workspace_bytes": (_sz, [_vp, _i, _i]),
    "gpt2_bind_memory": (_i, [_vp, _vp, _sz, _vp, _sz]),
    "gpt2_set_stream": (_i, [_vp, _vp]),
    "gpt2_forward": (_i, [_vp, _vp, _vp, _i, _i, _fp]),
    "gpt2_evaluate": (_i, [_vp, _vp, _vp, _i, _i, _fp]),
    "gpt2_set_recompute": (_i, [_vp, _i]),
    "gpt2_generate": (_i, [_vp, _vp, _i, _i, _i, _f, _i, _u64, _fp]),
    "gpt2_zero_grad": (_i, [_vp]),
    "gpt2_read_loss": (_i, [_vp, _fp]),
    "gpt2_backward": (_i, [_vp, _f]),
    "gpt2_grad_norm_clip": (_i, [_vp, _f, _fp]),
    "gpt2_adamw_step": (_i, [_vp, _f, _f, _f, _f, _f]),
    "gpt2_adamw_step_scheduled": (_i, [_vp, _d, _d, _l, _l, _f, _f, _f, _f]),
    "gpt2_step_graph_capture": (_i, [_vp, _vp, _vp, _i, _i, _i, _f, _d, _d, _l, _l, _f, _f, _f,
                                     _f]),
    "gpt2_step_graph_launch": (_i, [_vp]),
    "gpt2_padded_params": (_sz, [_vp]),
    "gpt2_grad_sumsq": (_i, [_vp, _sz, _sz, _vp]),
    "gpt2_clip_from_sumsq": (_i, [_vp, _vp, _f, _fp]),
    "gpt2_adamw_step_range": (_i, [_vp, _f, _f, _f, _f, _f, _sz, _sz]),
    "gpt2_params_device": (_i, [_vp, ctypes.POINTER(_fp)]),
    "gpt2_refresh_weights": (_i, [_vp]),
    "gpt2_set_backward_events": (_i, [_vp, ctypes.POINTER(_vp), _i]),
    "gpt2_step_graph_kernels": (_l, [_vp]),
    "gpt2_lr": (_d, [_l, _d, _d, _l, _l]),
    "gpt2_get_params": (_i, [_vp, _fp]),
    "gpt2_set_params": (_i, [_vp, _fp]),
    "gpt2_get_grads": (_i, [_vp, _fp]),
    "gpt2_get_state": (_i, [_vp, _fp, _fp, _fp, ctypes.POINTER(_l)]),
    "gpt2_set_state": (_i, [_vp, _fp, _fp, _fp, _l]),
    "gpt2_tensor_info": (_i, [_vp, _i, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(_i),
                              ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(_sz)]),
    "gpt2_logits": (_i, [_vp, ctypes.POINTER(_vp)]),
    "gpt2_grads_device": (_i, [_vp, ctypes.POINTER(_fp)]),
    "gpt2_get_losses": (_i, [_vp, _fp, _sz]),
    "gpt2_read_activation": (_i, [_vp, _i, _i, _fp, _sz]),
    "gpt2_last_error": (ctypes.c_char_p, [_vp]),
    "gpt2_launch_count": (_l, []),
    "gpt2_profile_enable": (_i, [_vp, _i]),
    "gpt2_profile_read": (_i, [_vp, ctypes.POINTER(_d), ctypes.POINTER(_l), ctypes.POINTER(_d), _i]),
    "gpt2k_gemm_set_cta_pairs": (_i, [_i]),
    "gpt2k_set_programmatic_launch": (_i, [_i]),
    "gpt2k_gemm": (_i, [_vp, _i, _i, _i, _i, _vp, _l, _i, _vp, _l, _i, _f, _vp, _l, _fp, _l, _fp,
                        _vp, _l, _vp, _l, _fp, _sz]),
    "gpt2k_attention_fwd": (_i, [_vp, _vp, _fp, _vp, _i, _i, _i, _i]),
    "gpt2k_attention_bwd_scratch": (_sz, [_i, _i, _i]),
    "gpt2k_attention_bwd": (_i, [_vp, _vp, _fp, _vp, _vp, _vp, _fp, _i, _i, _i, _i]),
    "gpt2k_layernorm_fwd": (_i, [_vp, _vp, _fp, _fp, _vp, _fp, _fp, _i, _i]),
    "gpt2k_layernorm_bwd": (_i, [_vp, _vp, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _fp, _fp, _i, _i, _i]),
    "gpt2k_layernorm_bwd_scratch": (_sz, [_i]),
    "gpt2k_classifier": (_i, [_vp, _vp, _fp, _vp, _i, _i, _i, _i]),
    "gpt2k_take_error": (_i, []),
    "gpt2k_gemm_expiry_test": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _i]),
    "gpt2k_gemm_wgrad_noalloc": (_i, [_vp, _i, _i, _i, _vp, _l, _vp, _l, _f, _fp, _l, _i, _vp]),
}

_LIBS: dict = {}


def lib_path(precision: str = "bf16") -> str:
    return os.path.join(LIBDIR, "libgpt2.so" if precision == "bf16" else "libgpt2_fp32.so")


def load(precision: str = "bf16") -> ctypes.CDLL:
    """Load the CUDA library; raises if it has not been built."""
    if precision in _LIBS:
        return _LIBS[precision]
    path = lib_path(precision)
    if not os.path.exists(path):
        raise RuntimeError(f"GPT-2 CUDA library not built: {path} is missing "
                           "(python -m transformer_lm_pretraining_b200.build)")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIBS[precision] = L
    return L


class GPT2Error(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


def _fptr(a: np.ndarray):
    assert a.dtype == np.float32 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_fp)


def _dptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


class GPT2:
    """One model + optimiser state on the current CUDA device."""

    def __init__(self, L, H, C, V, Vp, Tmax, seed=0, precision="bf16", B=None, T=None,
                 recompute=0):
        import torch

        self.torch = torch
        self.lib = load(precision)
        self.precision = precision
        self.cfg = (L, H, C, V, Vp, Tmax)
        h = _vp()
        rc = self.lib.gpt2_create(L, H, C, V, Vp, Tmax, seed, ctypes.byref(h))
        if rc:
            raise GPT2Error(rc, f"gpt2_create{(L, H, C, V, Vp, Tmax)}")
        self.h = h
        self.P = int(self.lib.gpt2_num_params(h))
        self._state = torch.empty(int(self.lib.gpt2_state_bytes(h)), dtype=torch.uint8, device="cuda")
        self._work = None
        self.set_stream()
        self._check(self.lib.gpt2_bind_memory(h, self._state.data_ptr(), self._state.numel(), None, 0))
        self._check(self.lib.gpt2_set_recompute(h, int(recompute)))
        if B is not None:
            self.reserve(B, T)

    def _check(self, rc):
        if rc:
            msg = self.lib.gpt2_last_error(self.h)
            raise GPT2Error(rc, msg.decode() if msg else "")
        return rc

    def close(self):
        if getattr(self, "h", None):
            self.torch.cuda.synchronize()
            self.lib.gpt2_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_stream(self, stream=None):
        s = stream if stream is not None else self.torch.cuda.current_stream()
        self._check(self.lib.gpt2_set_stream(self.h, s.cuda_stream))

    def workspace_bytes(self, B, T) -> int:
        return int(self.lib.gpt2_workspace_bytes(self.h, B, T))

    def reserve(self, B, T):
        need = self.workspace_bytes(B, T)
        if self._work is None or self._work.numel() < need:
            self._work = self.torch.empty(need, dtype=self.torch.uint8, device="cuda")
            self._check(self.lib.gpt2_bind_memory(self.h, None, 0, self._work.data_ptr(), need))

    # ---------------------------------------------------------------- step --
    def forward(self, tok, tgt=None, sync_loss=True):
        B, T = tok.shape
        self.reserve(B, T)
        out = ctypes.c_float(float("nan"))
        self._check(self.lib.gpt2_forward(self.h, _dptr(tok), _dptr(tgt), B, T,
                                          ctypes.byref(out) if sync_loss else None))
        return out.value if sync_loss else None

    def evaluate(self, tok, tgt, sync_loss=True):
        """Mean loss of a forward-only pass (no gradient is written, no
        backward may follow); perplexity = exp(loss)."""
        B, T = tok.shape
        self.reserve(B, T)
        out = ctypes.c_float(float("nan"))
        self._check(self.lib.gpt2_evaluate(self.h, _dptr(tok), _dptr(tgt), B, T,
                                           ctypes.byref(out) if sync_loss else None))
        return out.value if sync_loss else None

    def logits(self, B, T):
        """The logits buffer [B*T, Vpad] (a view into the workspace, activation
        dtype) after a forward without targets or an evaluation."""
        torch = self.torch
        ptr = ctypes.c_void_p()
        self._check(self.lib.gpt2_logits(self.h, ctypes.byref(ptr)))
        bf16 = self.precision == "bf16"

        class _View:  # CUDA array interface over the library's buffer
            __cuda_array_interface__ = {"shape": (B * T, self.cfg[4]), "typestr": "<i2" if bf16 else "<f4",
                                        "data": (ptr.value, False), "version": 2}

        t = torch.as_tensor(_View(), device="cuda")
        return t.view(torch.bfloat16) if bf16 else t

    def generate(self, tok, T_prompt, temperature=0.0, top_k=0, seed=0, step_logits=None):
        """Fill tok[:, T_prompt:] (a device int32 tensor [B, T_total]) by
        autoregressive generation with a key/value cache."""
        B, T_total = tok.shape
        self.reserve(B, T_prompt)
        sl = None if step_logits is None else ctypes.cast(ctypes.c_void_p(step_logits.data_ptr()), _fp)
        self._check(self.lib.gpt2_generate(self.h, _dptr(tok), B, T_prompt, T_total, temperature,
                                           top_k, seed, sl))

    def zero_grad(self):
        self._check(self.lib.gpt2_zero_grad(self.h))

    def read_loss(self):
        out = ctypes.c_float(float("nan"))
        self._check(self.lib.gpt2_read_loss(self.h, ctypes.byref(out)))
        return out.value

    def backward(self, loss_scale=1.0):
        self._check(self.lib.gpt2_backward(self.h, loss_scale))

    def grad_norm_clip(self, max_norm=1.0, sync=True):
        out = ctypes.c_float(float("nan"))
        self._check(self.lib.gpt2_grad_norm_clip(self.h, max_norm, ctypes.byref(out) if sync else None))
        return out.value if sync else None

    def adamw_step(self, lr, b1=0.9, b2=0.95, eps=1e-8, wd=0.1):
        self._check(self.lib.gpt2_adamw_step(self.h, lr, b1, b2, eps, wd))

    def adamw_step_scheduled(self, max_lr, min_lr, warmup, max_steps, b1=0.9, b2=0.95, eps=1e-8,
                             wd=0.1):
        self._check(self.lib.gpt2_adamw_step_scheduled(self.h, max_lr, min_lr, warmup, max_steps,
                                                       b1, b2, eps, wd))

    def capture_step(self, tok, tgt, B, T, n_micro, max_norm, max_lr, min_lr, warmup, max_steps,
                     b1=0.9, b2=0.95, eps=1e-8, wd=0.1):
        """Capture one optimizer step over the device token buffers tok, tgt
        (n_micro * B * T int32 each) as a CUDA graph; returns the number of
        kernels a replay runs."""
        self._check(self.lib.gpt2_step_graph_capture(self.h, _dptr(tok), _dptr(tgt), B, T, n_micro,
                                                     max_norm, max_lr, min_lr, warmup, max_steps,
                                                     b1, b2, eps, wd))
        return int(self.lib.gpt2_step_graph_kernels(self.h))

    def launch_step(self):
        """Replay the captured step on the model's stream (asynchronous)."""
        self._check(self.lib.gpt2_step_graph_launch(self.h))

    # ------------------------------------------------------------- state --
    def get_params(self) -> np.ndarray:
        a = np.empty(self.P, np.float32)
        self._check(self.lib.gpt2_get_params(self.h, _fptr(a)))
        return a

    def set_params(self, p):
        p = np.ascontiguousarray(p, np.float32)
        assert p.size == self.P
        self._check(self.lib.gpt2_set_params(self.h, _fptr(p)))

    def _device_view(self, getter, n):
        """A torch CUDA tensor over n fp32 elements of a library buffer (no copy)."""
        torch = self.torch
        ptr = _fp()
        self._check(getter(self.h, ctypes.byref(ptr)))
        addr = ctypes.cast(ptr, ctypes.c_void_p).value

        class _View:  # CUDA array interface over the library's buffer
            __cuda_array_interface__ = {"shape": (n,), "typestr": "<f4",
                                        "data": (addr, False), "version": 2}

        return torch.as_tensor(_View(), device="cuda")

    @property
    def padded_params(self) -> int:
        return int(self.lib.gpt2_padded_params(self.h))

    def grads_tensor(self, padded=False):
        """The model's fp32 gradient buffer [P] (or [padded_params] with the
        zero padding) as a torch CUDA tensor (a view, no copy): what replicas
        all-reduce, or reduce-scatter, between backward and clip."""
        return self._device_view(self.lib.gpt2_grads_device,
                                 self.padded_params if padded else self.P)

    def params_tensor(self, padded=False):
        """The fp32 parameter buffer as a torch CUDA tensor view (for the
        all-gather of updated shards; call refresh_weights afterwards)."""
        return self._device_view(self.lib.gpt2_params_device,
                                 self.padded_params if padded else self.P)

    def grad_sumsq(self, begin, end, out):
        """out (a float64 CUDA tensor of one element) = sum of squared
        gradients [begin, end)."""
        self._check(self.lib.gpt2_grad_sumsq(self.h, begin, end, _dptr(out)))

    def clip_from_sumsq(self, sumsq, max_norm=1.0, sync=True):
        out = ctypes.c_float(float("nan"))
        self._check(self.lib.gpt2_clip_from_sumsq(self.h, _dptr(sumsq), max_norm,
                                                  ctypes.byref(out) if sync else None))
        return out.value if sync else None

    def adamw_step_range(self, lr, b1, b2, eps, wd, begin, end):
        self._check(self.lib.gpt2_adamw_step_range(self.h, lr, b1, b2, eps, wd, begin, end))

    def refresh_weights(self):
        self._check(self.lib.gpt2_refresh_weights(self.h))

    def set_backward_events(self, events):
        """events: L + 1 torch.cuda.Event objects (recorded at least once, so
        that they exist) or None to stop recording."""
        if not events:
            self._check(self.lib.gpt2_set_backward_events(self.h, None, 0))
            return
        arr = (_vp * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
        self._check(self.lib.gpt2_set_backward_events(self.h, arr, len(events)))

    def get_grads(self) -> np.ndarray:
        a = np.empty(self.P, np.float32)
        self._check(self.lib.gpt2_get_grads(self.h, _fptr(a)))
        return a

    def get_state(self):
        p, m, v = (np.empty(self.P, np.float32) for _ in range(3))
        t = ctypes.c_long()
        self._check(self.lib.gpt2_get_state(self.h, _fptr(p), _fptr(m), _fptr(v), ctypes.byref(t)))
        return p, m, v, t.value

    def set_state(self, p, m, v, t):
        arrs = [np.ascontiguousarray(x, np.float32) for x in (p, m, v)]
        self._check(self.lib.gpt2_set_state(self.h, *[_fptr(x) for x in arrs], t))

    def tensor_info(self, i):
        name = ctypes.c_char_p()
        nd = ctypes.c_int()
        shape = (ctypes.c_int64 * 3)()
        off = ctypes.c_size_t()
        self._check(self.lib.gpt2_tensor_info(self.h, i, ctypes.byref(name), ctypes.byref(nd),
                                              shape, ctypes.byref(off)))
        return name.value.decode(), tuple(shape[: nd.value]), off.value

    def tensors(self):
        return [self.tensor_info(i) for i in range(16)]

    def get_losses(self, n):
        a = np.empty(n, np.float32)
        self._check(self.lib.gpt2_get_losses(self.h, _fptr(a), n))
        return a

    def profile_enable(self, on=True):
        self._check(self.lib.gpt2_profile_enable(self.h, int(on)))

    def profile_read(self):
        """{family: (ms, timed regions, algorithmic flops)}; clears the records."""
        n = len(PROF_KINDS)
        ms, cnt, fl = (ctypes.c_double * n)(), (ctypes.c_long * n)(), (ctypes.c_double * n)()
        self._check(self.lib.gpt2_profile_read(self.h, ms, cnt, fl, n))
        return {k: (ms[i], cnt[i], fl[i]) for i, k in enumerate(PROF_KINDS)}

    def read_activation(self, kind, layer, n):
        k = ACT_NAMES[kind] if isinstance(kind, str) else kind
        a = np.empty(n, np.float32)
        self._check(self.lib.gpt2_read_activation(self.h, k, layer, _fptr(a), n))
        return a


def gpt2_lr(step, max_lr, min_lr, warmup, max_steps, precision="bf16") -> float:
    return float(load(precision).gpt2_lr(step, max_lr, min_lr, warmup, max_steps))


def gpt2_launch_count(precision="bf16") -> int:
    return int(load(precision).gpt2_launch_count())


# ------------------------------------------------------ kernel-level calls --
def gpt2k_gemm_set_cta_pairs(enable, precision="bf16"):
    """Run wide products as 256 x 256 tiles over CTA pairs (1, the default)
    or as 128 x 256 tiles on single CTAs (0); returns the previous setting."""
    return load(precision).gpt2k_gemm_set_cta_pairs(1 if enable else 0)


def gpt2k_set_programmatic_launch(enable, precision="bf16"):
    """Programmatic dependent launch of the library's kernels on (1, the
    default) or off (0); returns the previous setting."""
    return load(precision).gpt2k_set_programmatic_launch(1 if enable else 0)


def gpt2k_gemm(epi, M, N, K, A, lda, a_mn, B, ldb, b_mn, alpha=1.0, out=None, ldo=0, out32=None,
               ldo32=0, bias=None, resid=None, ldr=0, aux=None, ldaux=0, split_ws=None,
               precision="bf16", stream=None):
    import torch

    L = load(precision)
    s = stream if stream is not None else torch.cuda.current_stream()
    e = EPI[epi] if isinstance(epi, str) else epi
    fp = lambda t: None if t is None else ctypes.cast(ctypes.c_void_p(t.data_ptr()), _fp)
    rc = L.gpt2k_gemm(s.cuda_stream, e, M, N, K, _dptr(A), lda, a_mn, _dptr(B), ldb, b_mn, alpha,
                      _dptr(out), ldo, fp(out32), ldo32, fp(bias), _dptr(resid), ldr, _dptr(aux),
                      ldaux, fp(split_ws), 0 if split_ws is None else split_ws.numel())
    if rc:
        raise GPT2Error(rc, "gpt2k_gemm")


def gpt2k_attention_fwd(att, lse, qkv, B, T, C, H, precision="bf16", stream=None):
    import torch

    L = load(precision)
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = L.gpt2k_attention_fwd(s.cuda_stream, _dptr(att), ctypes.cast(ctypes.c_void_p(lse.data_ptr()), _fp),
                               _dptr(qkv), B, T, C, H)
    if rc:
        raise GPT2Error(rc, "gpt2k_attention_fwd")


def gpt2k_attention_bwd_scratch(B, T, H, precision="bf16") -> int:
    """Floats of fp32 scratch gpt2k_attention_bwd needs."""
    return int(load(precision).gpt2k_attention_bwd_scratch(B, T, H))


def gpt2k_attention_bwd(dqkv, dsum, datt, qkv, att, lse, B, T, C, H, precision="bf16", stream=None):
    import torch

    L = load(precision)
    s = stream if stream is not None else torch.cuda.current_stream()
    cf = lambda t: ctypes.cast(ctypes.c_void_p(t.data_ptr()), _fp)
    rc = L.gpt2k_attention_bwd(s.cuda_stream, _dptr(dqkv), cf(dsum), _dptr(datt), _dptr(qkv),
                               _dptr(att), cf(lse), B, T, C, H)
    if rc:
        raise GPT2Error(rc, "gpt2k_attention_bwd")


def _f32p(t):
    return None if t is None else ctypes.cast(ctypes.c_void_p(t.data_ptr()), _fp)


def _stream(stream):
    import torch

    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def gpt2k_layernorm_fwd(y, mean, rstd, x, g, b, M, C, precision="bf16", stream=None):
    rc = load(precision).gpt2k_layernorm_fwd(_stream(stream), _dptr(y), _f32p(mean), _f32p(rstd),
                                             _dptr(x), _f32p(g), _f32p(b), M, C)
    if rc:
        raise GPT2Error(rc, "gpt2k_layernorm_fwd")


def gpt2k_layernorm_bwd_scratch(C, precision="bf16") -> int:
    return int(load(precision).gpt2k_layernorm_bwd_scratch(C))


def gpt2k_layernorm_bwd(dx, dy, x, mean, rstd, g, dg, db, dsum, partials, M, C, accumulate,
                        precision="bf16", stream=None):
    rc = load(precision).gpt2k_layernorm_bwd(
        _stream(stream), _dptr(dx), _dptr(dy), _dptr(x), _f32p(mean), _f32p(rstd), _f32p(g),
        _f32p(dg), _f32p(db), _f32p(dsum), _f32p(partials), M, C, 1 if accumulate else 0)
    if rc:
        raise GPT2Error(rc, "gpt2k_layernorm_bwd")


def gpt2k_classifier(logits, losses, tgt, M, V, Vp, write_grad=True, precision="bf16",
                     stream=None):
    rc = load(precision).gpt2k_classifier(_stream(stream), _dptr(logits), _f32p(losses),
                                          _dptr(tgt), M, V, Vp, 1 if write_grad else 0)
    if rc:
        raise GPT2Error(rc, "gpt2k_classifier")


def gpt2k_gemm_expiry_test(M, N, K, A, B, out, kblock=0, precision="bf16", stream=None) -> int:
    """The GEMM with one withheld k-block (test of the bounded waits);
    returns the C status."""
    return int(load(precision).gpt2k_gemm_expiry_test(_stream(stream), M, N, K, _dptr(A), _dptr(B),
                                                      _dptr(out), kblock))


def gpt2k_take_error(precision="bf16") -> int:
    return int(load(precision).gpt2k_take_error())


def gpt2k_gemm_wgrad_noalloc(M, N, K, A, lda, B, ldb, alpha, out32, ldo32, max_splits=8,
                             err=None, precision="bf16", stream=None) -> int:
    """Weight-gradient GEMM whose split-K scratch is the library's fixed
    device array (no device memory is allocated or passed in); returns the
    C status code (0 = OK)."""
    import torch

    L = load(precision)
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(L.gpt2k_gemm_wgrad_noalloc(
        s.cuda_stream, M, N, K, _dptr(A), lda, _dptr(B), ldb, alpha,
        ctypes.cast(ctypes.c_void_p(out32.data_ptr()), _fp), ldo32, max_splits, _dptr(err)))
