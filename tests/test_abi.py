"""Host-side checks of the C ABI (no GPU needed): the libraries load, export
every function the public headers declare, validate shapes, and their pure
host functions agree with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from transformer_lm_pretraining_b200 import gpt2 as g2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(gpt2k?_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module", params=["bf16", "fp32"])
def lib(request):
    if not os.path.exists(g2.lib_path(request.param)):
        from transformer_lm_pretraining_b200 import build
        build.build()
    return g2.load(request.param)


def test_headers_declare_the_step_calls():
    names = declared_functions()
    for want in ("gpt2_create", "gpt2_forward", "gpt2_backward", "gpt2_grad_norm_clip",
                 "gpt2_adamw_step", "gpt2_lr", "gpt2_zero_grad", "gpt2_bind_memory"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    missing = [n for n in sorted(names) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(g2.SIGNATURES) >= names


def test_build_flavour(lib):
    assert lib.gpt2_build_is_bf16() in (0, 1)
    assert g2.load("bf16").gpt2_build_is_bf16() == 1
    assert g2.load("fp32").gpt2_build_is_bf16() == 0


def _create(lib, *args):
    h = ctypes.c_void_p()
    rc = lib.gpt2_create(*args, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("args", [
    (12, 12, 768, 50257, 50257, 1024, 0),   # Vpad not a multiple of 64
    (12, 12, 768, 50257, 50240, 1024, 0),   # Vpad < V
    (2, 3, 128, 1024, 1024, 64, 0),         # C % H != 0
    (0, 4, 128, 1024, 1024, 64, 0),         # no layers
    (2, 4, 132, 1024, 1024, 64, 0),         # C % 8 != 0
])
def test_create_rejects_bad_shapes(lib, args):
    rc, h = _create(lib, *args)
    assert rc == -1 and not h.value


def test_param_count_and_layout_match_oracle(lib):
    for cfg in ((12, 12, 768, 50257, 50304, 1024), (2, 4, 128, 1024, 1024, 64),
                (8, 8, 512, 4096, 4096, 512)):
        rc, h = _create(lib, *cfg, 0)
        assert rc == 0
        L, H, C, V, Vp, Tmax = cfg
        o = oracle.Oracle(oracle.Config(*cfg))
        assert lib.gpt2_num_params(h) == o.num_params()
        assert lib.gpt2_num_params(h) == 12 * L * C * C + 13 * L * C + 2 * C + Vp * C + Tmax * C
        for i, (name, off, num, _) in enumerate(o.slices()):
            nm = ctypes.c_char_p()
            nd = ctypes.c_int()
            shape = (ctypes.c_int64 * 3)()
            o2 = ctypes.c_size_t()
            assert lib.gpt2_tensor_info(h, i, ctypes.byref(nm), ctypes.byref(nd), shape,
                                        ctypes.byref(o2)) == 0
            assert nm.value.decode() == name
            assert o2.value == off
            assert int(np.prod(shape[: nd.value])) == num
        # workspace grows with the batch
        assert lib.gpt2_workspace_bytes(h, 2, 64) > lib.gpt2_workspace_bytes(h, 1, 64) > 0
        assert lib.gpt2_state_bytes(h) >= (4 * 4 + (2 if lib.gpt2_build_is_bf16() else 0)) * o.num_params()
        lib.gpt2_destroy(h)


def test_lr_schedule_matches_oracle(lib):
    for step in (0, 1, 100, 714, 715, 716, 5000, 19073, 19074, 30000):
        a = lib.gpt2_lr(step, 6e-4, 6e-5, 715, 19073)
        b = oracle.lr(step, 6e-4, 6e-5, 715, 19073)
        assert a == pytest.approx(b, rel=1e-15, abs=0)
