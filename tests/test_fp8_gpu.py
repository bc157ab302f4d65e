"""GPU parity of the FP8 (E4M3) attention path.

Two checks per case:
  * the implementation: against the oracle's tiled model that rounds the
    weights to E4M3 the same way (per 128-key tile, lazy max with tau = 8),
    |O - O_model| <= 2^-8 |O_model| + 4e-3 (the bf16 output plus rare
    rounding flips where fp32 and fp64 weights fall on either side of an
    E4M3 rounding boundary), |LSE - LSE_exact| <= 1e-3 (l is kept in fp32);
  * the accuracy: against the exact definition on the same E4M3 inputs, a
    bound derived per output element from the E4M3 rounding of each weight.
    The kernel rounds p_j = 2^(x_j - m) (m its running maximum, log2 units)
    to E4M3 and divides by the unrounded sum l = sum_j p_j.  E4M3 keeps 3
    mantissa bits, so a weight in its normal range (p >= 2^-6) moves by at
    most 2^-4 p; below it the spacing is 2^-9, so it moves by at most
    min(p, 2^-10).  The lazy rule keeps m at or below the row's true
    maximum x_max, so l >= sum_j 2^(x_j - x_max) = 1 / w_max and, in the
    exact normalised weights w_j, |dw_j| <= max(2^-4 w_j, min(w_j,
    2^-10 w_max)).  Hence
    |O - O_exact| <= sum_j max(2^-4 w_j, min(w_j, 2^-10 w_max)) |v_j|
                     + 2^-8 |O_exact| + 2e-3
    (the last two terms: the bf16 output and the fp32 arithmetic).  A flip
    of the fp32 weight to the other E4M3 neighbour costs only the fp32
    error on top of the half spacing, so no factor is needed for it.
Descale factors are powers of two so the oracle sees the same values.
"""
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

pytestmark = pytest.mark.gpu


def run_case(oracle_mod, B, H, N, causal, seed, dq=0.5, dk=2.0, dv=0.25, q_std=1.0):
    d = 128
    scale = 1 / math.sqrt(d)
    q, k, v = make_qkv(B, H, N, d, seed, q_std)
    q8 = (q.float() / dq).to(torch.float8_e4m3fn)
    k8 = (k.float() / dk).to(torch.float8_e4m3fn)
    v8 = (v.float() / dv).to(torch.float8_e4m3fn)
    vt8 = v8.transpose(2, 3).contiguous()
    o, lse = tab.attn_fwd_fp8(q8.cuda(), k8.cuda(), vt8.cuda(), causal, scale, dq, dk, dv)
    assert tab.last_device_error() == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    # exact definition on the E4M3 values (exact in bf16; descales folded)
    qb, kb, vb = (bf16_bits(t.float().to(torch.bfloat16)) for t in (q8, k8, v8))
    o_ex, l_ex = oracle_mod.attn_ref(qb, kb, vb, causal, scale * dq * dk)
    o_ex = o_ex * dv
    Qd, Kd, Vd = (t.double().numpy() for t in (q8.float(), k8.float(), v8.float()))
    worst = []
    for b in range(B):
        for h in range(H):
            o_m, _ = oracle_mod.tiled_online_model(Qd[b, h], Kd[b, h], Vd[b, h], causal,
                                                   scale * dq * dk, round_p="e4m3")
            o_m = o_m * dv
            err = np.abs(o[b, h] - o_m)
            assert (err <= 2.0 ** -8 * np.abs(o_m) + 4e-3).all(), \
                f"b{b} h{h}: vs model max err {err.max():.3g}"
            S = Qd[b, h] @ Kd[b, h].T * (scale * dq * dk)
            if causal:
                S = np.where(np.tril(np.ones_like(S)) > 0, S, -np.inf)
            W = np.exp(S - S.max(1, keepdims=True))
            W /= W.sum(1, keepdims=True)
            dW = np.maximum(2.0 ** -4 * W, np.minimum(W, 2.0 ** -10 * W.max(1, keepdims=True)))
            bound = (dW @ np.abs(Vd[b, h])) * dv + 2.0 ** -8 * np.abs(o_ex[b, h]) + 2e-3
            err = np.abs(o[b, h] - o_ex[b, h])
            assert (err <= bound).all(), \
                f"b{b} h{h}: vs exact {int((err > bound).sum())} elements past the E4M3 bound"
            worst.append(float((err / np.maximum(bound, 1e-30)).max()))
    assert np.abs(lse - l_ex).max() <= 1e-3
    return max(worst)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 256, 640, 1024])
def test_fp8_matches_model_and_bound(oracle_mod, causal, N):
    run_case(oracle_mod, 1, 3, N, causal, seed=70 + N)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_ragged_and_peaky(oracle_mod, causal):
    run_case(oracle_mod, 2, 2, 400, causal, seed=91, q_std=3.0)


def test_fp8_rejects_unsupported_shapes():
    x = torch.zeros(1, 1, 100, 128, dtype=torch.uint8, device="cuda")
    vt = torch.zeros(1, 1, 128, 100, dtype=torch.uint8, device="cuda")
    with pytest.raises(tab.AttnError) as e:
        tab.attn_fwd_fp8(x, x, vt)  # N = 100 is not a multiple of 16
    assert e.value.status == -2
    x64 = torch.zeros(1, 1, 128, 64, dtype=torch.uint8, device="cuda")
    with pytest.raises(tab.AttnError):
        tab.attn_fwd_fp8(x64, x64, torch.zeros(1, 1, 64, 128, dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("N,d", [(256, 128), (1040, 64), (96, 128)])
def test_quantize_is_bit_exact(oracle_mod, transpose, N, d):
    """The conversion kernel's E4M3 bytes equal the oracle's codes (power-of
    -two scales: the fp32 and fp64 products agree), in either layout."""
    B, H = 2, 3
    x = make_qkv(B, H, N, d, seed=N + d)[0] * 3.0
    x = x.to(torch.bfloat16)
    for inv in (1.0, 8.0, 0.25):
        got = tab.quantize_e4m3(x.cuda(), inv, transpose).cpu().numpy()
        ref = oracle_mod.quantize_e4m3(bf16_bits(x), inv)
        if transpose:
            ref = np.ascontiguousarray(ref.transpose(0, 1, 3, 2))
        np.testing.assert_array_equal(got, ref)


def test_quantize_saturates_large_values(oracle_mod):
    x = torch.tensor([[1000.0, -1000.0, 447.0, 3e-4] * 32], dtype=torch.bfloat16)
    got = tab.quantize_e4m3(x.cuda(), 1.0).cpu().numpy()
    np.testing.assert_array_equal(got, oracle_mod.quantize_e4m3(bf16_bits(x), 1.0))
