"""GPU parity of the 4-bit (NVFP4) path: the conversion kernels and the
attention kernel.

The conversion (attn_quantize_nvfp4) must equal the oracle's quantisation
bit for bit: E2M1 codes and E4M3 scales, the scales in the tiled order the
block-scaled MMA reads them.

The attention (attn_fwd_fp4) is checked two ways on the same quantised
inputs (the oracle's own quantisation of the same bf16 draws):
  * the implementation: against the oracle's tiled model that rounds the
    weights to NVFP4 per 128-key tile and 16-key block under the lazy rule.
    The kernel's weights differ from the model's by the exponential's and
    the scale reciprocal's fp32 rounding, which can move a weight across an
    E2M1 or E4M3 rounding boundary; all but a few elements per thousand
    must agree to 2^-8 |O| + 4e-3, and every element must be within the
    derived bound below;
  * the accuracy: against the exact definition on the quantised inputs,
    |O - O_exact| <= sum_j dW_j |v_j| + 2^-8 |O_exact| + 2e-3 per element,
    dW_j the per-weight NVFP4 rounding bound that
    tests/test_oracle_fp4_pins.py derives and checks on the model.
  * LSE (from the unrounded fp32 row sum): within 1e-3 of the exact value.
"""
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

from test_oracle_fp4_pins import _weight_bound

pytestmark = pytest.mark.gpu


def pack_codes(c):
    """One E2M1 code per element -> two per byte, the lower-indexed element
    in the lower nibble."""
    c = np.asarray(c, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def tiled_scales(sc, n_rows):
    """Oracle scales [BH, rows, nblk] of an operand whose rows are the MMA's
    M/N rows and whose reduction axis is blocked by 16 -> the library's
    [BH, T, 2, 512] layout (reduction axis of 128 per tile; for Q and K the
    tile index runs over rows, nblk = 8)."""
    BH, R, nb = sc.shape
    T = (R + 127) // 128
    out = np.zeros((BH, T, 2, 512), dtype=np.uint8)
    for i in range(R):
        m = i % 128
        for kb in range(nb):
            out[:, i // 128, kb // 4, 16 * (m % 32) + 4 * (m // 32) + kb % 4] = sc[:, i, kb]
    return out


def tiled_scales_vt(sc, N):
    """Oracle scales of V^T [BH, 128 channels, N/16 key blocks] -> the
    [BH, T, 2, 512] layout (tiles over the keys, rows the channels)."""
    BH, C, nb = sc.shape
    T = (N + 127) // 128
    out = np.zeros((BH, T, 2, 512), dtype=np.uint8)
    for c in range(C):
        for kb in range(nb):
            out[:, kb // 8, (kb % 8) // 4, 16 * (c % 32) + 4 * (c // 32) + kb % 4] = sc[:, c, kb]
    return out


def oracle_quantize(oracle_mod, x, inv, transpose):
    """Oracle codes and tiled scales of bf16 x [B, H, N, 128]."""
    B, H, N, d = x.shape
    if transpose:
        xt = x.transpose(2, 3).contiguous().reshape(B * H, d, N)
        c, s = oracle_mod.quantize_nvfp4(bf16_bits(xt), inv)
        return pack_codes(c).reshape(B, H, d, N // 2), tiled_scales_vt(s, N), (c, s)
    c, s = oracle_mod.quantize_nvfp4(bf16_bits(x.reshape(B * H, N, d)), inv)
    return pack_codes(c).reshape(B, H, N, d // 2), tiled_scales(s, N), (c, s)


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("N", [96, 128, 320, 1024])
@pytest.mark.parametrize("inv", [1.0, 4.0, 0.25])
def test_quantize_nvfp4_is_bit_exact(oracle_mod, transpose, N, inv):
    B, H = 2, 3
    x = make_qkv(B, H, N, 128, seed=N + int(8 * inv), q_std=2.0)[0]
    codes, scales = tab.quantize_nvfp4(x.cuda(), inv, transpose)
    want_c, want_s, _ = oracle_quantize(oracle_mod, x, inv, transpose)
    np.testing.assert_array_equal(scales.cpu().numpy(), want_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), want_c)


def test_quantize_nvfp4_extremes(oracle_mod):
    """Large values saturate the scale, tiny ones give subnormal or zero
    scales, zero rows give zero scales."""
    x = torch.zeros(1, 1, 128, 128)
    x[0, 0, 0, :16] = 3072.0
    x[0, 0, 1, :16] = torch.linspace(-1e-3, 1e-3, 16)
    x[0, 0, 2, :] = torch.randn(128, generator=torch.Generator().manual_seed(1)) * 1e-4
    x = x.to(torch.bfloat16)
    for tr in (False, True):
        codes, scales = tab.quantize_nvfp4(x.cuda(), 1.0, tr)
        wc, ws, _ = oracle_quantize(oracle_mod, x, 1.0, tr)
        np.testing.assert_array_equal(scales.cpu().numpy(), ws)
        np.testing.assert_array_equal(codes.cpu().numpy(), wc)


def run_case(oracle_mod, B, H, N, causal, seed, q_std=1.0, dq=0.5, dk=2.0, dv=0.25):
    d = 128
    scale = 1 / math.sqrt(d)
    q, k, v = make_qkv(B, H, N, d, seed, q_std)
    qc, qs = tab.quantize_nvfp4(q.cuda(), 1 / dq, False)
    kc, ks = tab.quantize_nvfp4(k.cuda(), 1 / dk, False)
    vc, vs = tab.quantize_nvfp4(v.cuda(), 1 / dv, True)
    o, lse = tab.attn_fwd_fp4(qc, qs, kc, ks, vc, vs, causal, scale, dq, dk, dv)
    assert tab.last_device_error() == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    # the quantised inputs' values, from the oracle's own quantisation
    _, _, (c_q, s_q) = oracle_quantize(oracle_mod, q, 1 / dq, False)
    _, _, (c_k, s_k) = oracle_quantize(oracle_mod, k, 1 / dk, False)
    _, _, (c_v, s_v) = oracle_quantize(oracle_mod, v, 1 / dv, True)
    Qd = oracle_mod.nvfp4_to_f64(c_q, s_q).reshape(B, H, N, d)
    Kd = oracle_mod.nvfp4_to_f64(c_k, s_k).reshape(B, H, N, d)
    Vd = oracle_mod.nvfp4_to_f64(c_v, s_v).reshape(B, H, d, N).transpose(0, 1, 3, 2)
    sc = scale * dq * dk
    as_bits = lambda a: bf16_bits(torch.from_numpy(np.ascontiguousarray(a)).float().to(torch.bfloat16))
    o_ex, l_ex = oracle_mod.attn_ref(as_bits(Qd), as_bits(Kd), as_bits(Vd), causal, sc)
    o_ex = o_ex * dv
    tight_misses, worst = 0, 0.0
    for b in range(B):
        for h in range(H):
            o_m, _ = oracle_mod.tiled_online_model(Qd[b, h], Kd[b, h], Vd[b, h], causal, sc,
                                                   round_p="nvfp4")
            o_m = o_m * dv
            S = Qd[b, h] @ Kd[b, h].T * sc
            if causal:
                S = np.where(np.tril(np.ones_like(S)) > 0, S, -np.inf)
            W = np.exp(S - S.max(1, keepdims=True))
            W /= W.sum(1, keepdims=True)
            bound = (_weight_bound(W) @ np.abs(Vd[b, h])) * dv + 2.0 ** -8 * np.abs(o_ex[b, h]) \
                + 2e-3
            err = np.abs(o[b, h] - o_ex[b, h])
            assert (err <= bound).all(), \
                f"b{b} h{h}: {int((err > bound).sum())} elements past the NVFP4 bound"
            worst = max(worst, float((err / bound).max()))
            tight_misses += int((np.abs(o[b, h] - o_m) > 2.0 ** -8 * np.abs(o_m) + 4e-3).sum())
    assert tight_misses <= 2e-3 * o.size, f"{tight_misses} of {o.size} elements off the model"
    assert np.abs(lse - l_ex).max() <= 1e-3
    return worst, tight_misses


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [96, 128, 256, 640, 1024])
def test_fp4_matches_model_and_bound(oracle_mod, causal, N):
    run_case(oracle_mod, 1, 3, N, causal, seed=170 + N)


@pytest.mark.parametrize("causal", [False, True])
def test_fp4_peaky_scores(oracle_mod, causal):
    run_case(oracle_mod, 2, 2, 512, causal, seed=191, q_std=3.0)


def test_fp4_rejects_unsupported_shapes():
    x = torch.zeros(1, 1, 100, 64, dtype=torch.uint8, device="cuda")
    sf = torch.zeros(1, 1, 2, 512, dtype=torch.uint8, device="cuda")
    vt = torch.zeros(1, 1, 128, 50, dtype=torch.uint8, device="cuda")
    with pytest.raises(tab.AttnError) as e:
        tab.attn_fwd_fp4(x, sf, x, sf, vt, sf)  # N = 100 is not a multiple of 32
    assert e.value.status == -2
    with pytest.raises(tab.AttnError) as e:
        tab.quantize_nvfp4(torch.zeros(1, 1, 100, 128, dtype=torch.bfloat16, device="cuda"),
                           1.0, True)
    assert e.value.status == -2
