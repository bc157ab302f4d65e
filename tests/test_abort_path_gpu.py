"""The attention kernels' abort path, run without any fault.

Every wait inside the kernels is bounded: a wait that runs out records
ATTN_ERR_DEVICE_TIMEOUT in the device status word and raises the CTA's abort
flag; every role then leaves its loop, the producer waits (bounded) for its
loads in flight, the MMA warp for its products in flight, and Tensor Memory
is freed (page lecompute.fr/en/kernel-perf/flapping-airplanes-thunderkittens-
megakernels, section "A persistent program takes responsibility for
progress").

The test library (libattn_b200_testhooks.so, ATTN_TEST_HOOKS) adds one entry
point: a shorter wait limit and the index of one K/V tile load that the
producer of CTA 0 skips.  The consumer of that tile then waits until its
limit runs out.  Nothing faults, traps or waits without end.  Checked for the
two-tile kernel (d = 128), the wide kernel (d = 256) and the FP8 kernel:
  * the call returns and the status word reads the timeout once, then 0;
  * the next launch on the same GPU matches the oracle, which it could not
    do if Tensor Memory had been left allocated (its allocation would not
    be granted on that SM).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from tiled_attention_forward_sm_b200 import build as tab_build
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000  # 5 ms


@pytest.fixture(scope="module")
def hooks():
    lib = ctypes.CDLL(tab_build.build_test_hooks())
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd.argtypes = [vp] * 5 + [i] * 5 + [f, vp]
    lib.attn_fwd.restype = i
    lib.attn_fwd_fp8.argtypes = [vp] * 5 + [i] * 5 + [f, f, f, f, vp]
    lib.attn_fwd_fp8.restype = i
    lib.attn_test_set_hooks.argtypes = [ctypes.c_ulonglong, i]
    lib.attn_test_set_hooks.restype = i
    lib.attn_last_device_error.argtypes = [vp]
    lib.attn_last_device_error.restype = i
    yield lib
    lib.attn_test_set_hooks(0, -1)


def _run_bf16(lib, q, k, v, causal, scale):
    B, H, N, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    rc = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, H, N, d, int(causal), scale, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return o, lse


def _status(lib):
    return lib.attn_last_device_error(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("withhold", [0, 1])  # loads every first item has
def test_withheld_load_times_out_and_the_next_launch_is_correct(oracle_mod, hooks, d, withhold,
                                                                causal):
    """Without the mask (and at d = 256 always) the other CTAs' epilogues
    leave through TMA stores while CTA 0 aborts; every CTA waits for its
    stores to read their staging boxes before it exits."""
    scale = 1 / math.sqrt(d)
    B, H, N = 1, 4, 1024
    qh, kh, vh = make_qkv(B, H, N, d, seed=500 + d + withhold)
    q, k, v = (t.cuda() for t in (qh, kh, vh))
    assert hooks.attn_test_set_hooks(LIMIT_NS, withhold) == 0
    _run_bf16(hooks, q, k, v, causal, scale)
    assert _status(hooks) == -5  # ATTN_ERR_DEVICE_TIMEOUT, read and cleared
    assert _status(hooks) == 0
    assert hooks.attn_test_set_hooks(LIMIT_NS, -1) == 0
    o, lse = _run_bf16(hooks, q, k, v, causal, scale)
    assert _status(hooks) == 0
    o_ref, l_ref = oracle_mod.attn_ref(bf16_bits(qh), bf16_bits(kh), bf16_bits(vh), causal, scale)
    o64 = o.double().cpu().numpy()
    assert (np.abs(o64 - o_ref) <= 2e-2 + 1e-2 * np.abs(o_ref)).all()
    assert np.abs(lse.double().cpu().numpy() - l_ref).max() <= 1e-3


@pytest.mark.parametrize("causal", [True, False])
def test_fp8_withheld_load_times_out_and_the_next_launch_runs(oracle_mod, hooks, causal):
    B, H, N, d = 1, 4, 1024, 128
    q, k, v = make_qkv(B, H, N, d, seed=77)
    q8, k8 = (t.float().to(torch.float8_e4m3fn).cuda() for t in (q, k))
    vt8 = v.float().to(torch.float8_e4m3fn).transpose(2, 3).contiguous().cuda()
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream

    def run():
        return hooks.attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), vt8.data_ptr(), o.data_ptr(),
                                  lse.data_ptr(), B, H, N, d, int(causal), 1 / math.sqrt(d), 1.0,
                                  1.0, 1.0, s)
    assert hooks.attn_test_set_hooks(LIMIT_NS, 1) == 0
    assert run() == 0
    assert _status(hooks) == -5
    assert _status(hooks) == 0
    assert hooks.attn_test_set_hooks(LIMIT_NS, -1) == 0
    assert run() == 0
    assert _status(hooks) == 0
    # the exact definition on the E4M3 inputs, within the loose FP8 bound
    qb, kb, vb = (bf16_bits(t.float().to(torch.float8_e4m3fn).float().to(torch.bfloat16))
                  for t in (q, k, v))
    o_ex, l_ex = oracle_mod.attn_ref(qb, kb, vb, causal, 1 / math.sqrt(d))
    assert np.abs(lse.double().cpu().numpy() - l_ex).max() <= 1e-3
    assert np.abs(o.double().cpu().numpy() - o_ex).max() <= 0.25
