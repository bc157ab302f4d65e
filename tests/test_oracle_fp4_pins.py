"""Pins of the oracle's 4-bit (NVFP4) functions, CPU only.

NVFP4: E2M1 elements (sign, 2 exponent bits with bias 1, 1 mantissa bit)
with one E4M3 scale per 16 consecutive elements.  The pins do not go
through the oracle's own code paths:
  * the E2M1 value of every code against a hand-written table
    (tests/golden/nvfp4_examples.json, from the format's definition);
  * rounding against a brute-force search over the representable values
    with ties to the even mantissa;
  * whole blocks worked by hand (scale rounding, saturation of the scale
    and of the elements, a subnormal scale, an all-zero block, negative
    zeros);
  * invariants: each element lands on one of the two E2M1 neighbours of
    x / scale (or saturates), scaling by powers of two moves only the
    scale, negation flips only the sign bits;
  * the tiled model with NVFP4-rounded weights stays inside a bound
    derived from the rounding of each weight, and uses a visible part of it.
"""
import json
import os

import numpy as np
import pytest
import torch

from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_examples.json")
MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _bits(values):
    x = torch.tensor(values, dtype=torch.float32)
    assert torch.equal(x.to(torch.bfloat16).float(), x)
    return bf16_bits(x.to(torch.bfloat16))


def test_e2m1_decode_matches_the_hand_table(oracle_mod):
    g = _golden()["e2m1_values"]
    codes = np.arange(16, dtype=np.uint8)
    got = oracle_mod.e2m1_bits_to_f64(codes)
    want = np.array([g[str(c)] for c in range(16)])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(want))  # -0 for code 8


def _brute_round(x):
    """Nearest representable magnitude by exhaustive search; a tie goes to
    the even mantissa (the table index's low bit is the mantissa)."""
    out = np.empty_like(x)
    for i, v in enumerate(x):
        a = min(abs(v), 6.0)
        d = np.abs(MAGS - a)
        best = np.flatnonzero(d == d.min())
        k = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        out[i] = -MAGS[k] if np.signbit(v) else MAGS[k]
    return out


def test_e2m1_rounding_matches_brute_force(oracle_mod):
    rng = np.random.default_rng(3)
    mids = (MAGS[1:] + MAGS[:-1]) / 2
    x = np.concatenate([rng.uniform(-8, 8, 20000), mids, -mids, MAGS, -MAGS, [6.5, -7.0, 100.0]])
    np.testing.assert_array_equal(oracle_mod.round_e2m1(x), _brute_round(x))


def test_e2m1_encoding_round_trips_every_code(oracle_mod):
    codes = np.arange(16, dtype=np.uint8)
    vals = oracle_mod.e2m1_bits_to_f64(codes)
    np.testing.assert_array_equal(oracle_mod.e2m1_encode(vals), codes)
    with pytest.raises(ValueError):
        oracle_mod.e2m1_encode(np.array([0.75]))


@pytest.mark.parametrize("k", range(4))
def test_hand_worked_blocks(oracle_mod, k):
    b = _golden()["blocks"][k]
    codes, sc = oracle_mod.quantize_nvfp4(_bits(b["x"])[None, :], 1.0)
    assert int(sc[0, 0]) == b["scale_code"], b["what"]
    assert oracle_mod.e4m3_bits_to_f64(sc)[0, 0] == b["scale"]
    assert list(codes[0]) == b["codes"], b["what"]


def test_block_invariants(oracle_mod):
    x = make_qkv(2, 3, 64, 128, 8, q_std=2.0)[0]
    bits = bf16_bits(x)
    codes, sc = oracle_mod.quantize_nvfp4(bits, 1.0)
    xf = x.float().numpy().astype(np.float64)
    s = oracle_mod.e4m3_bits_to_f64(sc)
    v = oracle_mod.e2m1_bits_to_f64(codes)
    blk = lambda a: a.reshape(a.shape[:-1] + (a.shape[-1] // 16, 16))
    # the scale is amax / 6 rounded to E4M3 (a relative half-step of 2^-4)
    amax = np.abs(blk(xf)).max(-1)
    assert (np.abs(s - amax / 6) <= 2.0 ** -4 * amax / 6 + 2.0 ** -10).all()
    # each element is one of the two E2M1 neighbours of x / s, or saturated
    t = blk(xf) / s[..., None]
    lo = np.array([MAGS[MAGS <= a].max() for a in np.minimum(np.abs(t), 6).ravel()])
    hi = np.array([MAGS[MAGS >= a].min() for a in np.minimum(np.abs(t), 6).ravel()])
    a = np.abs(blk(v)).ravel()
    assert ((a == lo) | (a == hi)).all()
    # powers of two move only the scale
    for e in (-3, 2):
        c2, s2 = oracle_mod.quantize_nvfp4(bf16_bits((x.float() * 2.0 ** e).to(torch.bfloat16)), 1.0)
        np.testing.assert_array_equal(c2, codes)
        np.testing.assert_array_equal(oracle_mod.e4m3_bits_to_f64(s2), s * 2.0 ** e)
    # negation flips only the sign bits
    c3, s3 = oracle_mod.quantize_nvfp4(bf16_bits(-x), 1.0)
    np.testing.assert_array_equal(c3, codes ^ 0x8)
    np.testing.assert_array_equal(s3, sc)
    # inv_descale is applied before quantising, exactly for powers of two
    c4, s4 = oracle_mod.quantize_nvfp4(bits, 0.25)
    np.testing.assert_array_equal(c4, codes)
    np.testing.assert_array_equal(oracle_mod.e4m3_bits_to_f64(s4), s * 0.25)


def _weight_bound(W):
    """Per-weight bound on |dW| for NVFP4-rounded softmax weights (rows of
    exact normalised weights W, blocks of 16 keys from key 0).  In units of
    the kernel's running scale a block's scale s = E4M3(pmax / 6) and an
    element moves by at most a quarter of max(p, s) inside the E2M1 range,
    plus what saturation at 6 s costs when s rounded down: at most
    max(6 * 2^-10, 2^-4 pmax).  The lazy maximum keeps the running sum at
    least 1 / w_max, so absolute terms in those units are at most
    (term) * w_max once normalised."""
    n = W.shape[1]
    pad = (-n) % 16
    Wp = np.pad(W, ((0, 0), (0, pad)))
    blk = Wp.reshape(W.shape[0], -1, 16)
    bmax = blk.max(-1, keepdims=True)
    wmax = W.max(1, keepdims=True)[:, :, None]
    s = bmax / 6 * (1 + 2.0 ** -4) + 2.0 ** -10 * wmax
    sat = np.maximum(6 * 2.0 ** -10 * wmax, 2.0 ** -4 * bmax)
    dW = 0.25 * np.maximum(blk, s) + sat
    return dW.reshape(W.shape[0], -1)[:, :n]


def test_model_with_nvfp4_weights_stays_inside_its_bound(oracle_mod):
    def q4(t):
        c, s = oracle_mod.quantize_nvfp4(bf16_bits(t[0, 0]), 1.0)
        return oracle_mod.nvfp4_to_f64(c, s)
    for q_std, seed, n in ((1.0, 5, 512), (3.0, 6, 400)):
        q, k, v = make_qkv(1, 1, n, 128, seed, q_std)
        Q, K = q4(q), q4(k)
        # V is quantised along the keys (the second product's reduction axis)
        cv, sv = oracle_mod.quantize_nvfp4(bf16_bits(v[0, 0].t().contiguous()), 1.0)
        V = oracle_mod.nvfp4_to_f64(cv, sv).T
        scale = 128 ** -0.5
        for causal in (False, True):
            o_ex, _ = oracle_mod.tiled_online_model(Q, K, V, causal, scale)
            o_m, _ = oracle_mod.tiled_online_model(Q, K, V, causal, scale, round_p="nvfp4")
            S = Q @ K.T * scale
            if causal:
                S = np.where(np.tril(np.ones_like(S)) > 0, S, -np.inf)
            W = np.exp(S - S.max(1, keepdims=True))
            W /= W.sum(1, keepdims=True)
            bound = _weight_bound(W) @ np.abs(V)
            err = np.abs(o_m - o_ex)
            assert (err <= bound * (1 + 1e-9) + 1e-12).all()
            assert (err / np.maximum(bound, 1e-30)).max() > 0.05
