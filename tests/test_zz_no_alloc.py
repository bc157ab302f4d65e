"""The allocation-free entry point, attn_fwd_noalloc.

It is meant for callers that cannot allocate device memory (for example code
running under global-mode CUDA stream capture, where cudaMalloc is refused,
or inside a framework whose allocator owns all device memory).  It runs the
same kernel as attn_fwd with its work-queue scratch in the library's fixed
device array, cleared on every call.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 2e-2, 1e-2, 1e-3


def _noalloc_call(lib, q, k, v, o, lse, causal, scale):
    B, H, N, d = q.shape
    return lib.attn_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, H, N, d, int(causal), ctypes.c_float(scale),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("causal,shape", [(True, (2, 4, 1024, 128)), (False, (1, 3, 640, 64)),
                                          (True, (1, 2, 384, 64)), (True, (1, 2, 300, 96))])
def test_noalloc_matches_attn_fwd_on_two_calls_in_a_row(causal, shape):
    B, H, N, d = shape
    scale = 1.0 / d ** 0.5
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=4242 + N + d))
    o_ref, lse_ref = tab.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert tab.last_device_error() == 0
    lib = tab.library()
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(lib, q, k, v, o, lse, causal, scale) == 0
        assert tab.last_device_error() == 0
        o64, r64 = o.double().cpu().numpy(), o_ref.double().cpu().numpy()
        assert np.isfinite(o64).all() and torch.isfinite(lse).all()
        assert (np.abs(o64 - r64) <= ATOL_O + RTOL_O * np.abs(r64)).all(), f"call {call}: O"
        assert (lse - lse_ref).abs().max().item() <= ATOL_LSE, f"call {call}: LSE"


def test_noalloc_rejects_bad_arguments_like_attn_fwd():
    lib = tab.library()
    q = torch.zeros(1, 1, 128, 80, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    o = torch.zeros_like(q)
    assert _noalloc_call(lib, q, q, q, o, lse, False, 0.1) == -2  # d = 80 is unsupported
    assert tab.last_device_error() == 0
