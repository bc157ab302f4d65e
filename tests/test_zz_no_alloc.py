"""The allocation-free entry point, attn_fwd_noalloc.

Some callers of this library cannot allocate device memory: a framework
whose caching allocator has already reserved the GPU's memory (a cudaMalloc
would fail, or force the cache to be released), or a serving loop that has
fixed its memory budget at start-up and must not let cudaMalloc's implicit
device synchronisation into its hot path.  attn_fwd_noalloc runs the same
kernel as attn_fwd, with the work-queue counter in the library's fixed
device array, cleared on every call.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes
import gc
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

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
                                          (True, (1, 2, 384, 64)), (True, (1, 2, 300, 96)),
                                          (False, (1, 2, 640, 256)), (True, (1, 3, 520, 256))])
def test_noalloc_matches_attn_fwd_on_two_calls_in_a_row(oracle_mod, causal, shape):
    """Two calls in a row through the C ABI: each bitwise equal to attn_fwd
    (the same kernel on the same inputs; the results do not depend on which
    CTA takes which work item) and within the parity tolerance of the
    oracle.  d = 256 runs the wide kernel on the same scratch counter."""
    B, H, N, d = shape
    scale = 1.0 / math.sqrt(d)
    qh, kh, vh = make_qkv(B, H, N, d, seed=4242 + N + d)
    q, k, v = (t.cuda() for t in (qh, kh, vh))
    o_ref, lse_ref = tab.attn_fwd(q, k, v, causal=causal, scale=scale)
    assert tab.last_device_error() == 0
    o_or, l_or = oracle_mod.attn_ref(bf16_bits(qh), bf16_bits(kh), bf16_bits(vh), causal, scale)
    lib = tab.library()
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc_call(lib, q, k, v, o, lse, causal, scale) == 0
        assert tab.last_device_error() == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"call {call}: not bitwise"
        o64 = o.double().cpu().numpy()
        assert (np.abs(o64 - o_or) <= ATOL_O + RTOL_O * np.abs(o_or)).all(), f"call {call}: O"
        assert np.abs(lse.double().cpu().numpy() - l_or).max() <= ATOL_LSE, f"call {call}: LSE"


@pytest.mark.parametrize("d", [128, 256])
def test_noalloc_takes_no_device_memory(d):
    """After a first call on the device (which sets the library up), further
    calls leave the device's free memory and torch's allocation unchanged."""
    B, H, N = 1, 4, 1024
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=77))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    lib = tab.library()
    scale = 1.0 / math.sqrt(d)
    assert _noalloc_call(lib, q, k, v, o, lse, True, scale) == 0
    torch.cuda.synchronize()
    # tensors of earlier tests that the garbage collector frees would move
    # the counters: collect first, and not while measuring
    gc.collect()
    gc.disable()
    try:
        free0, _ = torch.cuda.mem_get_info()
        alloc0 = torch.cuda.memory_allocated()
        for _ in range(3):
            assert _noalloc_call(lib, q, k, v, o, lse, True, scale) == 0
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        alloc1 = torch.cuda.memory_allocated()
    finally:
        gc.enable()
    assert alloc1 == alloc0
    assert free1 == free0
    assert tab.last_device_error() == 0


def test_noalloc_rejects_bad_arguments_like_attn_fwd():
    lib = tab.library()
    q = torch.zeros(1, 1, 128, 80, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, dtype=torch.float32, device="cuda")
    o = torch.zeros_like(q)
    assert _noalloc_call(lib, q, q, q, o, lse, False, 0.1) == -2  # d = 80 is unsupported
    assert tab.last_device_error() == 0


@pytest.mark.parametrize("causal,d", [(True, 128), (False, 128), (False, 256)])
def test_noalloc_captured_in_a_cuda_graph(causal, d):
    """attn_fwd_noalloc inside stream capture (torch.cuda.graph, global
    capture mode): after a first call on the device, the call captures a
    memset of the scratch counter and the kernel, and each replay on new
    contents of the same buffers equals attn_fwd bitwise."""
    B, H, N = 1, 4, 1000
    scale = 1.0 / math.sqrt(d)
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=900 + d))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    lib = tab.library()
    assert _noalloc_call(lib, q, k, v, o, lse, causal, scale) == 0  # first call: device set-up
    torch.cuda.synchronize()
    assert tab.last_device_error() == 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rc = _noalloc_call(lib, q, k, v, o, lse, causal, scale)
    assert rc == 0
    for trial in range(3):
        qn, kn, vn = make_qkv(B, H, N, d, seed=910 + d + trial)
        q.copy_(qn)
        k.copy_(kn)
        v.copy_(vn)
        o.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert tab.last_device_error() == 0
        o_ref, l_ref = tab.attn_fwd(q, k, v, causal=causal, scale=scale)
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref), f"replay {trial}"
    del graph


def test_attn_fwd_captured_in_a_cuda_graph():
    """attn_fwd itself also captures after a first call on the device: the
    launch takes its work-queue slot at capture time, every replay reuses
    it, and the launch's last CTA resets it, so replays in stream order stay
    correct (bitwise equal to eager calls)."""
    B, H, N, d, causal = 2, 4, 2048, 128, True
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, seed=930))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    tab.attn_fwd_into(q, k, v, o, lse, causal=causal)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        tab.attn_fwd_into(q, k, v, o, lse, causal=causal)
    for trial in range(3):
        for dst, src in zip((q, k, v), make_qkv(B, H, N, d, seed=931 + trial)):
            dst.copy_(src)
        graph.replay()
        torch.cuda.synchronize()
        assert tab.last_device_error() == 0
        o_ref, l_ref = tab.attn_fwd(q, k, v, causal=causal)
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref), f"replay {trial}"
    del graph
