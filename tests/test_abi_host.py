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


@pytest.mark.parametrize("d", [64, 96, 128, 256])
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
    assert tab.check_args(*p, 1, 1, 128, 80, 0.1) == -2                # d unsupported
    assert tab.check_args(*p, 1, 1, 128, 32, 0.1) == -2                # d unsupported
    assert tab.check_args(*p, 1, 1, 128, 512, 0.1) == -2               # d unsupported
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
        opts = tab.AttnOpts(bad, 0)
        rc = lib.attn_fwd_ex(*p, 1, 1, 128, 128, 0, 0.1, ctypes.byref(opts), None)
        assert rc == -1
    for bad in (-1, 1, 6):  # ring depths
        opts = tab.AttnOpts(-1, bad)
        assert lib.attn_fwd_ex(*p, 1, 1, 128, 128, 0, 0.1, ctypes.byref(opts), None) == -1
    # depths other than the default only at d = 128 with the default split
    assert lib.attn_fwd_ex(*p, 1, 1, 128, 64, 0, 0.1, ctypes.byref(tab.AttnOpts(-1, 3)), None) == -2
    assert lib.attn_fwd_ex(*p, 1, 1, 128, 128, 0, 0.1, ctypes.byref(tab.AttnOpts(1, 3)), None) == -2
    for bad in (-0.5, 16.5, float("nan"), float("inf")):  # rescale thresholds
        opts = tab.AttnOpts(-1, 0, bad)
        assert lib.attn_fwd_ex(*p, 1, 1, 128, 128, 0, 0.1, ctypes.byref(opts), None) == -1
    assert lib.attn_fwd_ex(*p, 1, 1, 128, 256, 0, 0.1, ctypes.byref(tab.AttnOpts(-1, 0, 4.0)),
                           None) == -2
    d = lib.attn_opts_default()
    assert (d.exp2_poly_pairs, d.kv_stages, d.rescale_tau) == (-1, 0, -1.0)


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


def test_exp2_degree5_polynomial_of_the_fp8_kernel():
    """The FP8 kernel's degree-5 literals are the generator's, and the fp32
    sequence stays within 2.5e-7 relative of 2^x (about ex2.approx's own
    error), so E4M3 rounding of the weights flips no more often."""
    import importlib.util
    import numpy as np
    gen_path = os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc", "gen_exp2_poly.py")
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", gen_path)
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c = [float(np.float32(v)) for v in gen.remez_relative(5)]
    src = open(os.path.join(ROOT, "tiled_attention_forward_sm_b200", "csrc",
                            "attn_fwd_fp8_kernel.cuh")).read()
    lits = [float(x) for x in re.findall(r"kE[0-5] = ([0-9.]+)f", src)]
    assert len(lits) == 6
    assert np.allclose(lits, c, rtol=0, atol=1e-10)
    xs = np.linspace(-125.0, 8.0, 400001).astype(np.float32)
    rel = np.abs(gen.fp32_exp2_emulation(xs, lits).astype(np.float64) /
                 np.exp2(xs.astype(np.float64)) - 1.0)
    assert rel.max() < 2.5e-7


def test_trace_reader_knows_the_kernel_events():
    """The trace reader takes its event list from the kernel source."""
    from tiled_attention_forward_sm_b200 import trace
    names = trace.event_names()
    assert names[0] == "MmaS0" and "Sm1Pb" in names and "End" in names
    assert len(names) == len(set(names)) == 24


def test_selftest_rejects_bad_limit(lib):
    assert lib.attn_selftest_wait_timeout(0, None) == -1
    assert lib.attn_selftest_wait_timeout(-5, None) == -1
    assert lib.attn_selftest_wait_timeout(20000000, None) == -1


def test_new_entry_points_are_declared():
    syms = declared_symbols()
    for s in ["attn_fwd_chunk", "attn_fwd_varlen", "attn_fwd_splitkv", "attn_combine",
              "attn_fwd_noalloc", "attn_selftest_wait_timeout"]:
        assert s in syms


def test_chunk_rejections_before_any_cuda_call(lib):
    """attn_fwd_chunk's host checks (no device needed to reach them)."""
    q, k, v, o, l = ptrs()
    f = lib.attn_fwd_chunk
    ok = (1, 4, 2, 128, 256, 128, 1, 128, 0.1, 0)
    assert f(q, k, v, o, l, 1, 4, 3, 128, 256, 128, 1, 0, 0.1, 0, None) == -1  # H % H_kv
    assert f(q, k, v, o, l, 1, 4, 0, 128, 256, 128, 1, 0, 0.1, 0, None) == -1  # H_kv = 0
    assert f(q, k, v, o, l, 1, 4, 2, 0, 256, 128, 1, 0, 0.1, 0, None) == -1    # N_q = 0
    assert f(q, k, v, o, l, 1, 4, 2, 128, 0, 128, 1, 0, 0.1, 0, None) == -1    # N_k = 0
    assert f(q, k, v, o, l, 1, 4, 2, 128, 256, 80, 1, 0, 0.1, 0, None) == -2   # d
    assert f(q, k, v, o, l, 1, 4, 2, 128, 256, 128, 1, (1 << 30) + 1, 0.1, 0, None) == -1
    assert f(q + 8, k, v, o, l, 1, 4, 2, 128, 256, 128, 1, 0, 0.1, 0, None) == -3
    # LSE placed right after a bf16 O of 4*128 rows: fine for a bf16 O (the
    # call then fails only for want of a device), an overlap for an fp32 O
    big = A + (1 << 28)
    ob = 4 * 128 * 128 * 2
    args = (big, big + (1 << 22), big + (1 << 23), big + (1 << 24), big + (1 << 24) + ob,
            1, 4, 2, 128, 256, 128, 1, 0, 0.1)
    assert f(*args, 0, None) not in (-1, -2, -3)
    assert f(*args, 1, None) == -1
    del ok


def test_varlen_rejections_before_any_cuda_call(lib):
    q, k, v, o, l = ptrs()
    cq, ck = A + (1 << 26), A + (1 << 26) + 4096
    f = lib.attn_fwd_varlen
    base = (q, k, v, o, l, cq, ck)
    assert f(*base[:5], 0, ck, 2, 4, 2, 64, 64, 100, 100, 128, 1, 0.1, None) == -1  # null offsets
    assert f(*base, 0, 4, 2, 64, 64, 100, 100, 128, 1, 0.1, None) == -1   # B = 0
    assert f(*base, 2, 4, 3, 64, 64, 100, 100, 128, 1, 0.1, None) == -1   # H % H_kv
    assert f(*base, 2, 4, 2, 0, 64, 100, 100, 128, 1, 0.1, None) == -1    # max_seqlen_q
    assert f(*base, 2, 4, 2, 64, 64, 0, 100, 128, 1, 0.1, None) == -1     # total_q
    assert f(*base, 2, 4, 2, 64, 64, 100, 100, 96 + 16, 1, 0.1, None) == -2
    assert f(*base, 2, 4, 2, 64, 64, 100, 100, 128, 1, float("nan"), None) == -1
    assert f(q, k, v, o, l, cq + 2, ck, 2, 4, 2, 64, 64, 100, 100, 128, 1, 0.1, None) == -3
    assert f(q, k, v, o, l, cq, o, 2, 4, 2, 64, 64, 100, 100, 128, 1, 0.1, None) == -1  # cu_k in o
    assert f(*base, 2, 1 << 16, 1, 64, 64, 1 << 15, 1 << 15, 128, 1, 0.1, None) == -2  # rows


def test_splitkv_and_combine_rejections_before_any_cuda_call(lib):
    q, k, v, o, l = ptrs(128, 1, 1, 1024)
    w_o, w_l = A + (1 << 27), A + (1 << 28)
    f = lib.attn_fwd_splitkv
    g = (1, 1, 1, 1024, 1024, 128, 1, 0, 0.1)
    assert f(q, k, v, o, l, *g, 0, w_o, w_l, None) == -1     # 0 slices
    assert f(q, k, v, o, l, *g, 257, w_o, w_l, None) == -1   # too many
    assert f(q, k, v, o, l, *g, 4, None, w_l, None) == -1    # no scratch
    assert f(q, k, v, o, l, *g, 4, w_o + 4, w_l, None) == -3
    assert f(q, k, v, o, l, *g, 4, q, w_l, None) == -1       # scratch = q
    assert f(q, k, v, o, l, 1, 2, 3, 1024, 1024, 128, 1, 0, 0.1, 4, w_o, w_l, None) == -1  # heads
    c = lib.attn_combine
    assert c(w_o, w_l, 0, 100, 128, o, l, 0, None) == -1      # G = 0
    assert c(w_o, w_l, 2, 0, 128, o, l, 0, None) == -1        # rows = 0
    assert c(w_o, w_l, 2, 100, 80, o, l, 0, None) == -2       # d
    assert c(w_o + 8, w_l, 2, 100, 128, o, l, 0, None) == -3
    assert c(w_o, w_l, 2, 100, 128, w_o, l, 0, None) == -1    # output over a part


def test_kmeans_rejections_before_any_cuda_call(lib):
    f = lib.attn_kmeans_assign
    x, c, ws, a_, b_ = A, A + (1 << 24), A + (1 << 25), A + (1 << 26), A + (1 << 27)
    assert f(None, c, ws, a_, b_, 1000, 64, 128, None) == -1
    assert f(x, c, ws, a_, b_, 0, 64, 128, None) == -1          # N = 0
    assert f(x, c, ws, a_, b_, 1000, 0, 128, None) == -1        # K = 0
    assert f(x, c, ws, a_, b_, 1000, 64, 96, None) == -2        # d
    assert f(x + 8, c, ws, a_, b_, 1000, 64, 128, None) == -3   # misaligned x
    assert f(x, c, ws, a_ + 2, b_, 1000, 64, 128, None) == -3   # misaligned assign
    assert f(x, c, x, a_, b_, 1000, 64, 128, None) == -1        # scratch over the points
    assert lib.attn_kmeans_workspace_floats(1000, 64) == 128 + 1000
    assert lib.attn_kmeans_workspace_floats(1000, 129) == 256 + 1000
    assert lib.attn_kmeans_workspace_floats(0, 5) == -1


def test_fp8_rejections_before_any_cuda_call(lib):
    q, k, v, o, l = ptrs(128, 1, 1, 1024)
    f = lib.attn_fwd_fp8
    good = (1, 1, 1024, 128, 1, 0.1, 1.0, 1.0, 1.0)
    assert f(q, k, v, o, l, 1, 1, 1000, 128, 1, 0.1, 1.0, 1.0, 1.0, None) == -2   # N % 16
    assert f(q, k, v, o, l, 1, 1, 1024, 64, 1, 0.1, 1.0, 1.0, 1.0, None) == -2    # d
    assert f(q, k, v, o, l, 1, 1, 1024, 128, 1, 0.1, 0.0, 1.0, 1.0, None) == -1   # descale
    assert f(q, k, v, o, l, 1, 1, 1024, 128, 1, 0.1, 1.0, 1.0, float("nan"), None) == -1
    assert f(q + 8, k, v, o, l, *good, None) == -3
    assert f(q, k, v, q, l, *good, None) == -1                                    # o over q


def test_quantize_rejections_before_any_cuda_call(lib):
    f = lib.attn_quantize_e4m3
    s, d_ = A, A + (1 << 26)
    assert f(None, d_, 1, 128, 128, 1.0, 0, None) == -1
    assert f(s, d_, 1, 128, 96, 1.0, 0, None) == -2         # d
    assert f(s, d_, 1, 100, 128, 1.0, 1, None) == -2        # transposed N % 16
    assert f(s, d_, 1, 128, 128, 0.0, 0, None) == -1        # scale
    assert f(s + 8, d_, 1, 128, 128, 1.0, 0, None) == -3
    assert f(s, s + 64, 1, 128, 128, 1.0, 0, None) == -1    # overlap


def test_pair_rejections_before_any_cuda_call(lib):
    q, k, v, o, l = ptrs(128, 1, 1, 1024)
    f = lib.attn_fwd_pair
    assert "attn_fwd_pair" in declared_symbols()
    assert f(q, k, v, o, l, 1, 1, 1024, 64, 1, 0.1, None) == -2                  # d
    assert f(q, k, v, o, l, 1, 1, 1024, 96, 0, 0.1, None) == -2
    assert f(q, k, v, o, l, 0, 1, 1024, 128, 1, 0.1, None) == -1                 # B
    assert f(q, k, v, o, l, 1, 1, 1024, 128, 1, float("inf"), None) == -1       # scale
    assert f(q + 8, k, v, o, l, 1, 1, 1024, 128, 1, 0.1, None) == -3
    assert f(q, k, v, o, l + 2, 1, 1, 1024, 128, 1, 0.1, None) == -3
    assert f(q, k, v, q, l, 1, 1, 1024, 128, 1, 0.1, None) == -1                 # o over q
    assert f(None, k, v, o, l, 1, 1, 1024, 128, 1, 0.1, None) == -1


def test_binding_requires_one_cuda_device():
    """The binding resolves the one device every tensor lives on and runs the
    call with it current; tensors on two devices, or not on a GPU, are
    refused before the library is called."""
    import torch
    from tiled_attention_forward_sm_b200 import _abi
    cpu = torch.zeros(4)
    meta = torch.zeros(4, device="meta")
    with pytest.raises(ValueError, match="one CUDA device"):
        _abi._device_of(cpu, meta)
    with pytest.raises(ValueError, match="CUDA tensors"):
        _abi._device_of(cpu, cpu)
    with pytest.raises(ValueError, match="CUDA tensors"):
        _abi._device_of(None, cpu, None)  # None entries are skipped


def test_product_library_carries_no_test_hooks(lib):
    """The abort-path hooks exist only in the test library."""
    assert not hasattr(lib, "attn_test_set_hooks")
    if os.path.exists(tab_build.TEST_HOOKS_LIB):
        import ctypes
        assert hasattr(ctypes.CDLL(tab_build.TEST_HOOKS_LIB), "attn_test_set_hooks")
