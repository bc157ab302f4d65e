"""Host-side tests of the C ABI: the library loads without a GPU, exports
every symbol include/attn_b200.h declares, and rejects bad arguments before
any CUDA call."""
import math
import os
import re

import pytest

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200 import build as tab_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    tab_build.build()
    return tab.library()


def declared_symbols():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_entry_points():
    syms = declared_symbols()
    for s in ["attn_fwd", "attn_fwd_ex", "attn_fwd_host", "attn_last_device_error",
              "attn_strerror", "attn_check_args", "attn_version"]:
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), f"{s} declared in include/ but not exported"


def test_strerror_and_version(lib):
    assert tab.strerror(0) == "ok"
    for code in (-1, -2, -3, -4, -5, -7, 12345):
        assert isinstance(tab.strerror(code), str) and tab.strerror(code)
    assert lib.attn_version() > 0


A = 1 << 20  # a 16-byte aligned fake address; check_args never dereferences


def ptrs(d=128, B=1, H=1, N=128):
    tb = B * H * N * d * 2
    return [A, A + tb, A + 2 * tb, A + 3 * tb, A + 4 * tb]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 256, 384, 1000, 32768])
def test_check_args_accepts_supported(lib, d, N):
    assert tab.check_args(*ptrs(d, 2, 3, N), 2, 3, N, d, 1 / math.sqrt(d)) == 0


def test_check_args_rejections(lib):
    p = ptrs()
    assert tab.check_args(0, *p[1:], 1, 1, 128, 128, 0.1) == -1        # null q
    assert tab.check_args(*p[:4], 0, 1, 1, 128, 128, 0.1) == -1        # null lse
    assert tab.check_args(*p, 0, 1, 128, 128, 0.1) == -1               # B = 0
    assert tab.check_args(*p, 1, -1, 128, 128, 0.1) == -1              # H < 0
    assert tab.check_args(*p, 1, 1, 0, 128, 0.1) == -1                 # N = 0
    assert tab.check_args(*p, 1, 1, 128, 128, 0.0) == -1               # scale 0
    assert tab.check_args(*p, 1, 1, 128, 128, -1.0) == -1              # scale < 0
    assert tab.check_args(*p, 1, 1, 128, 128, float("nan")) == -1
    assert tab.check_args(*p, 1, 1, 128, 128, float("inf")) == -1
    assert tab.check_args(*p, 1, 1, 128, 96, 0.1) == -2                # d unsupported
    assert tab.check_args(*p, 1, 1, 128, 256, 0.1) == -2               # d unsupported
    assert tab.check_args(*p, 1 << 12, 1 << 12, 1 << 8, 128, 0.1) == -2  # rows >= 2^31
    q, k, v, o, l = p
    assert tab.check_args(q + 8, k, v, o, l, 1, 1, 128, 128, 0.1) == -3   # misaligned q
    assert tab.check_args(q, k, v, o + 2, l, 1, 1, 128, 128, 0.1) == -3   # misaligned o
    assert tab.check_args(q, k, v, o, l + 2, 1, 1, 128, 128, 0.1) == -3   # misaligned lse
    assert tab.check_args(q, k, v, q, l, 1, 1, 128, 128, 0.1) == -1       # o aliases q
    assert tab.check_args(q, k, v, o, v + 64, 1, 1, 128, 128, 0.1) == -1  # lse inside v
    assert tab.check_args(q, q, q, o, l, 1, 1, 128, 128, 0.1) == 0        # inputs may alias


def test_binding_rejects_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        tab.attn_fwd(x, x, x)


def test_product_does_not_import_oracle():
    """The product package never imports or names the oracle."""
    pkg = os.path.join(ROOT, "tiled_attention_forward_sm_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), fn
                assert "attn_ref" not in text and "libattn_ref" not in text, fn


def test_fwd_ex_rejects_bad_option_before_any_cuda_call(lib):
    import ctypes
    p = ptrs()
    for bad in (-2, 3, 100):
        opts = tab.AttnOpts(bad)
        rc = lib.attn_fwd_ex(*p, 1, 1, 128, 128, 0, 0.1, ctypes.byref(opts), None)
        assert rc == -1


def test_exp2_polynomial_coefficients_and_error():
    """The kernel's exp2 polynomial literals are the ones the generator
    derives, and the fp32 instruction sequence stays within 1e-4 relative
    error of 2^x over the clamped range (far below bf16's 2^-9)."""
    import importlib.util
    import numpy as np
    gen_path = os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc", "gen_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", gen_path)
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c = [float(np.float32(v)) for v in gen.remez_relative()]
    src = open(os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc",
                            "attn_fwd_kernel.cuh")).read()
    lits = [float(x) for x in re.findall(r"kC[0-3] = ([0-9.]+)f", src)]
    # every copy (packed and scalar forms) carries the derived coefficients
    assert len(lits) >= 4 and len(lits) % 4 == 0
    for k in range(0, len(lits), 4):
        assert np.allclose(lits[k:k + 4], c, rtol=0, atol=1e-9)
    lits = lits[:4]
    xs = np.linspace(-125.0, 8.0, 400001).astype(np.float32)
    rel = np.abs(gen.fp32_exp2_emulation(xs, lits).astype(np.float64) /
                 np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    # integers are exact up to the polynomial's value at f = 0
    ints = np.arange(-125, 9).astype(np.float32)
    np.testing.assert_allclose(gen.fp32_exp2_emulation(ints, lits), np.exp2(ints) * lits[0],
                               rtol=1e-7)


def test_selftest_rejects_bad_limit(lib):
    assert lib.attn_selftest_wait_timeout(0, None) == -1
    assert lib.attn_selftest_wait_timeout(-5, None) == -1
    assert lib.attn_selftest_wait_timeout(20000000, None) == -1
