"""CPU checks of the constructed lazy-rescale inputs (inputs.make_jump_qkv).

The GPU test that uses them (tests/test_parity_gpu.py,
test_lazy_rescale_at_known_rows) is only as strong as the construction, so
this file checks, on the exact bf16 values, that:
  * every row's running maximum jumps by exactly the intended amount at the
    intended K/V tile (more than the bf16 kernels' default threshold, just
    under it, or not at all), in both 128-row Q tiles of a work item and
    under the causal mask;
  * a lazy-rescale step with a plausible mistake (the rescale factor's sign
    flipped, the rescale of O skipped, or applied to the other Q tile's rows)
    moves the result outside the parity tolerance at those rows, while the
    correct step stays inside it.

The lazy rule is the one of page lecompute.fr/kernel-perf/flashattention-4-
limites-calcul-matriciel, section "Deplacer une partie des exponentielles":
a common scale kept between old and new contributions, some rescalings
skipped under a condition.  The planted mistakes live in a copy of the
tiled step written here, on the CPU; the oracle itself is not changed.
"""
import math

import numpy as np
import pytest

from tiled_attention_forward_sm_b200.inputs import (DEFAULT_RESCALE_TAU, JUMP_OFFSETS, bf16_bits,
                                                    jump_offset_of_rows, make_jump_qkv)

ATOL_O, RTOL_O = 2e-2, 1e-2
TAU = DEFAULT_RESCALE_TAU
UNDER = JUMP_OFFSETS[1]  # the jump just under the threshold
SCALE = math.log(2.0)  # scale * log2(e) = 1: raw scores are log2 units


def _f64(t):
    return t.double().numpy()


def _tiled(q, k, v, causal, mistake=None):
    """The tiled online softmax with the lazy rule, fp64, one (b, h); with a
    planted mistake when asked.  Returns O."""
    N = q.shape[0]
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    acc = np.zeros_like(q)
    rows = np.arange(N)
    for j0 in range(0, N, 128):
        cols = np.arange(j0, min(j0 + 128, N))
        x = q @ k[cols].T  # log2 units (scale * log2 e = 1)
        if causal:
            x = np.where(cols[None, :] <= rows[:, None], x, -np.inf)
        tmax = x.max(1)
        up = (tmax - m) > TAU
        new_m = np.where(up, tmax, m)
        with np.errstate(invalid="ignore"):
            alpha = np.where(up, np.exp2(m - new_m), 1.0)
        alpha = np.where(np.isneginf(m), 0.0, alpha)
        if mistake == "alpha_sign":
            alpha = np.where(up & np.isfinite(m), np.exp2(new_m - m), alpha)
        p = np.where(np.isneginf(x), 0.0, np.exp2(x - new_m[:, None]))
        l = l * alpha + p.sum(1)
        a_o = alpha
        if mistake == "skip_o_rescale":
            a_o = np.where(np.isneginf(m), 0.0, 1.0)
        elif mistake == "other_tile":
            # the factor of row r applied to row r +- 128 (the other Q tile of
            # the pair), as if the two softmax groups' O regions were swapped
            a_o = alpha.copy()
            for t0 in range(0, N - 128, 256):
                a, b = slice(t0, t0 + 128), slice(t0 + 128, min(t0 + 256, N))
                n_b = b.stop - b.start
                tmp = a_o[a][:n_b].copy()
                a_o[a][:n_b] = alpha[b]
                a_o[b] = tmp
        acc = acc * a_o[:, None] + p @ v[cols]
        m = new_m
    return acc / l[:, None]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("jump_tile,second", [(1, False), (2, True)])
def test_jump_rows_take_the_intended_branch(causal, jump_tile, second):
    N, d = 640, 64
    q, k, v = make_jump_qkv(1, 2, N, d, jump_tile, second, seed=5)
    c = jump_offset_of_rows(N)
    for h in range(2):
        Q, K = _f64(q[0, h]), _f64(k[0, h])
        S = Q @ K.T
        rows = np.arange(N)
        if causal:
            S = np.where(np.arange(N)[None, :] <= rows[:, None], S, -np.inf)
        before = S[:, : 128 * jump_tile].max(1)
        at = S[:, 128 * jump_tile: 128 * (jump_tile + 1)].max(1)
        assert (before == 2.0).all()  # the anchor is every row's max so far
        sees = rows >= 128 * jump_tile if causal else np.ones(N, bool)
        np.testing.assert_array_equal(at[sees], 2.0 + c[sees])
        assert (at[~sees] == -np.inf).all() or not causal
        # both branches occur in both Q tiles of some work item
        taken = sees & (at - before > TAU)
        under = sees & (c == UNDER)
        assert UNDER < TAU < JUMP_OFFSETS[0]
        assert (at[under] - before[under] == UNDER).all()
        pair_rows = [(rows // 128) % 2 == s for s in (0, 1)]
        for s in (0, 1):
            assert (taken & pair_rows[s]).any() and (under & pair_rows[s]).any()
        # and within single warps both branches occur, and warps with one
        warp = rows // 32
        mixed = [w for w in np.unique(warp[sees]) if
                 taken[warp == w].any() and (sees & ~taken)[warp == w].any()]
        assert mixed
    assert set(np.unique(c)) == set(JUMP_OFFSETS)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("mistake", ["alpha_sign", "skip_o_rescale", "other_tile"])
def test_planted_rescale_mistakes_leave_the_tolerance(oracle_mod, causal, mistake):
    N, d = 640, 64
    q, k, v = make_jump_qkv(1, 1, N, d, 2, True, seed=6)
    o_ref, _ = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, SCALE)
    o_ref = o_ref[0, 0]
    Q, K, V = _f64(q[0, 0]), _f64(k[0, 0]), _f64(v[0, 0])
    good = _tiled(Q, K, V, causal)
    np.testing.assert_allclose(good, o_ref, rtol=1e-10, atol=1e-12)
    bad = _tiled(Q, K, V, causal, mistake)
    out = np.abs(bad - o_ref) > ATOL_O + RTOL_O * np.abs(o_ref)
    assert out.any(), f"planted mistake {mistake} stays inside the tolerance"


def test_default_threshold_matches_the_kernel():
    """The inputs' threshold mirrors the bf16 kernels' default (the constant
    in the kernel source), so the constructed jumps straddle the threshold
    the product uses."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(__file__), "..", "tiled_attention_forward_sm_b200",
                            "csrc", "attn_fwd_kernel.cuh")).read()
    value = float(re.search(r"constexpr float kRescaleTauBf16 = ([0-9.]+)f;", src).group(1))
    assert value == DEFAULT_RESCALE_TAU
