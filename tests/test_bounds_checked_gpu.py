"""The bounds-checked debug build (libattn_b200_checked.so).

Built with ATTN_BOUNDS_CHECKS, the kernels check every tensor-map coordinate
(the first row or token of each Q, K and V tile, and its head) and every O
and LSE store index against the extents of the launch's tensors before the
access is issued.  A failed check writes ATTN_ERR_DEVICE_BOUNDS to the
status word, raises the CTA's abort flag and skips the access; nothing
traps.  This is the debug-build form of race and overrun detection for the
buffer-reuse hazards of page lecompute.fr/en/kernel-perf/flapping-airplanes-
thunderkittens-megakernels, section "Prepare the next operation without
overwriting the current one".

  * On every layout the product supports (dense, ragged N, causal, d 64 to
    256, query and key lengths apart, shared K/V heads, key slices, packed
    variable lengths) the checked build reports no violation and returns
    bitwise the product library's results: the checks are silent on correct
    work and change no arithmetic.
  * With the test hook that adds an offset to the K/V head of CTA 0's first
    work item (a head past the end of K and V), the check fires before any
    load of that head: the status word reads ATTN_ERR_DEVICE_BOUNDS, and the
    next launch is correct again.  The tensor maps would only have filled
    such a tile with zeros, so nothing here can fault.
"""
import contextlib
import ctypes
import math

import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200 import _abi
from tiled_attention_forward_sm_b200 import build as tab_build
from tiled_attention_forward_sm_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

ATTN_ERR_DEVICE_BOUNDS = -6


@pytest.fixture(scope="module")
def checked():
    lib = _abi.configure(ctypes.CDLL(tab_build.build_checked()))
    lib.attn_test_set_bad_kv_head.argtypes = [ctypes.c_int]
    lib.attn_test_set_bad_kv_head.restype = ctypes.c_int
    yield lib
    lib.attn_test_set_bad_kv_head(0)


@contextlib.contextmanager
def through(lib):
    """Route the binding's calls through another build of the library."""
    saved = _abi._lib
    _abi._lib = lib
    try:
        yield
    finally:
        _abi._lib = saved


def both(checked, fn):
    """fn() through the product library and through the checked build:
    both results, after checking that neither reported a device error."""
    ref = fn()
    assert tab.last_device_error() == 0
    with through(checked):
        got = fn()
        status = tab.last_device_error()
    assert status == 0, f"checked build reported {status}"
    return ref, got


def assert_bitwise(ref, got):
    for r, g in zip(ref, got):
        assert torch.equal(r, g)


@pytest.mark.parametrize("B,H,N,d,causal,q_std", [
    (2, 4, 1024, 128, True, 1.0), (1, 3, 1000, 128, False, 1.0), (1, 2, 777, 64, True, 1.0),
    (1, 2, 640, 96, False, 2.0), (1, 2, 300, 256, True, 1.0), (8, 16, 512, 128, False, 3.0),
    (1, 1, 1, 128, True, 1.0)])
def test_checked_build_is_silent_and_bitwise_on_dense_layouts(checked, B, H, N, d, causal, q_std):
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=N + d, q_std=q_std))
    ref, got = both(checked, lambda: tab.attn_fwd(q, k, v, causal=causal))
    assert_bitwise(ref, got)


@pytest.mark.parametrize("causal", [False, True])
def test_checked_build_on_chunks_and_shared_kv_heads(checked, causal):
    B, H, H_kv, N_q, N_k, d = 2, 8, 2, 384, 1536, 128
    g = torch.Generator().manual_seed(11)
    q = torch.randn(B, H, N_q, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H_kv, N_k, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H_kv, N_k, d, generator=g).to(torch.bfloat16).cuda()
    ref, got = both(checked, lambda: tab.attn_fwd_chunk(q, k, v, causal=causal,
                                                        causal_delta=N_k - N_q))
    assert_bitwise(ref, got)


def test_checked_build_on_key_slices(checked):
    B, H, H_kv, N_q, N_k, d = 2, 8, 2, 128, 4096, 128
    g = torch.Generator().manual_seed(12)
    q = torch.randn(B, H, N_q, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, H_kv, N_k, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H_kv, N_k, d, generator=g).to(torch.bfloat16).cuda()
    ref, got = both(checked, lambda: tab.attn_fwd_splitkv(q, k, v, 4, causal=True,
                                                          causal_delta=N_k - N_q))
    assert_bitwise(ref, got)


@pytest.mark.parametrize("causal", [False, True])
def test_checked_build_on_packed_variable_lengths(checked, causal):
    lens = [1, 130, 500, 1024, 77]
    H, H_kv, d = 4, 2, 128
    T = sum(lens)
    g = torch.Generator().manual_seed(13)
    q = torch.randn(T, H, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(T, H_kv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(T, H_kv, d, generator=g).to(torch.bfloat16).cuda()
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32).cuda()
    ref, got = both(checked, lambda: tab.attn_fwd_varlen(q, k, v, cu, cu, max(lens), max(lens),
                                                         causal=causal))
    assert_bitwise(ref, got)


@pytest.mark.parametrize("d", [128, 256])
def test_planted_bad_kv_head_is_caught_before_the_load(checked, d):
    B, H, N = 1, 4, 1024
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=900 + d))
    ref = tab.attn_fwd(q, k, v, causal=True)
    assert tab.last_device_error() == 0
    with through(checked):
        assert checked.attn_test_set_bad_kv_head(1 << 20) == 0
        try:
            tab.attn_fwd(q, k, v, causal=True)
            first = tab.last_device_error()
            again = tab.last_device_error()
        finally:
            assert checked.attn_test_set_bad_kv_head(0) == 0
        assert first == ATTN_ERR_DEVICE_BOUNDS
        assert again == 0  # reading the status clears it
        got = tab.attn_fwd(q, k, v, causal=True)
        assert tab.last_device_error() == 0
    assert_bitwise(ref, got)
