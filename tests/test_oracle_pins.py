"""Pins for the CPU oracle: closed forms, special cases, invariants and brute
force that do not go through the oracle's own code.

The definition pinned is the one on page lecompute.fr/kernel-perf/
flashattention-4-limites-calcul-matriciel, section "Entre deux
multiplications il faut fabriquer les poids" (scores, softmax weights that are
positive and sum to one, a second product mixing V), with the causal reading
"key j visible to query i iff j <= i" (section "Le FP4 ajoute un compromis
numerique").  Each test names the mistake it is there to catch.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_bits(x) -> np.ndarray:
    """float array -> bf16 bits; asserts every value is exactly bf16."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "fixture value not representable in bf16"
    return bf16_bits(b)


def f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _const(s: str) -> float:
    table = {"0": 0.0, "ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4),
             "ln7": math.log(7), "ln7/4": math.log(7 / 4)}
    return table[s]


# ---------------------------------------------------------------- golden ---
@pytest.mark.parametrize("causal", [False, True])
def test_hand_examples(oracle_mod, causal):
    """Hand-derived weights that are simple fractions (tests/golden)."""
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = to_bits(np.array(c["q"])[None, None])
        k = to_bits(np.array(c["k"])[None, None])
        v = to_bits(np.array(c["v"])[None, None])
        o, lse = oracle_mod.attn_ref(q, k, v, causal, _const(c["scale"]))
        exp = c["causal" if causal else "noncausal"]
        np.testing.assert_allclose(o[0, 0], np.array(exp["o"]), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, 0], [_const(s) for s in exp["lse"]], rtol=0, atol=1e-14)


# ------------------------------------------------------------ invariants ---
@pytest.mark.parametrize("causal", [False, True])
def test_row_weights_sum_to_one(oracle_mod, causal):
    """Weights exp(s_ij - LSE_i) are >= 0 and sum to 1 over visible keys.
    Catches a wrong LSE (missing max, wrong log base, missing scale)."""
    B, H, N, d = 2, 3, 37, 16
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=11))
    scale = 0.37
    _, lse = oracle_mod.attn_ref(q, k, v, causal, scale)
    Q, K = f64(q), f64(k)
    s = np.einsum("bhid,bhjd->bhij", Q, K) * scale
    if causal:
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    w = np.exp(s - lse[..., None])
    assert (w >= 0).all()
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean_of_v(oracle_mod, causal):
    """Q = 0: all scores equal, O_i = mean of the visible V rows and
    LSE_i = log |J_i|.  Catches a wrong mask extent or a wrong normaliser."""
    B, H, N, d = 1, 2, 23, 8
    _, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=12))
    q = np.zeros_like(k)
    o, lse = oracle_mod.attn_ref(q, k, v, causal, 0.5)
    V = f64(v)
    for i in range(N):
        J = i + 1 if causal else N
        np.testing.assert_allclose(o[:, :, i], V[:, :, :J].mean(axis=2), rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], math.log(J), rtol=0, atol=1e-13)


def test_dominating_score_selects_its_value_row(oracle_mod):
    """One score 64 above the rest: O_i = V[j*] to 1e-12 and LSE_i = that
    score (plus a log(1 + (N-1)e^-64) term below 1e-25).  Catches a
    transposed operand or a key/value row mismatch."""
    N, d = 16, 8
    _, _, v = (bf16_bits(t) for t in make_qkv(1, 1, N, d, seed=13))
    V = f64(v)[0, 0]
    for i, jstar in [(0, 5), (7, 7), (15, 2)]:
        q = np.zeros((1, 1, N, d)); k = np.zeros((1, 1, N, d))
        q[0, 0, i, 0] = 8.0
        k[0, 0, jstar, 0] = 8.0
        o, lse = oracle_mod.attn_ref(to_bits(q), to_bits(k), v, False, 1.0)
        np.testing.assert_allclose(o[0, 0, i], V[jstar], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, 0, i], 64.0, rtol=0, atol=1e-12)


def test_causal_row0_is_v0(oracle_mod):
    """Causal row 0 sees only key 0: O_0 = V_0 exactly, LSE_0 = scale q0.k0.
    Catches an off-by-one in the mask (j < i instead of j <= i)."""
    B, H, N, d = 2, 2, 40, 16
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=14))
    scale = 1 / math.sqrt(d)
    o, lse = oracle_mod.attn_ref(q, k, v, True, scale)
    Q, K, V = f64(q), f64(k), f64(v)
    np.testing.assert_array_equal(o[:, :, 0], V[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * (Q[:, :, 0] * K[:, :, 0]).sum(-1), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_single_key(oracle_mod, causal):
    """N = 1: O = V and LSE = scale q.k.  Catches a missing scale."""
    B, H, N, d = 3, 2, 1, 64
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=15))
    o, lse = oracle_mod.attn_ref(q, k, v, causal, 0.125)
    np.testing.assert_array_equal(o, f64(v))
    np.testing.assert_allclose(lse, 0.125 * (f64(q) * f64(k)).sum(-1), rtol=0, atol=1e-13)


# ----------------------------------------------------------- brute force ---
def _brute_long_double(Q, K, V, causal, scale):
    """exp(s)/sum exp(s) with no max subtraction, in long double, written
    independently of the oracle (plain loops)."""
    N, d = Q.shape
    ld = np.longdouble
    o = np.zeros((N, d), dtype=ld); lse = np.zeros(N, dtype=ld)
    for i in range(N):
        J = range(i + 1) if causal else range(N)
        e = []
        for j in J:
            s = ld(0)
            for c in range(d):
                s += ld(Q[i, c]) * ld(K[j, c])
            e.append(np.exp(ld(scale) * s))
        tot = ld(0)
        for x in e:
            tot += x
        for jj, j in enumerate(J):
            for c in range(d):
                o[i, c] += e[jj] * ld(V[j, c]) / tot
        lse[i] = np.log(tot)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (5, 3), (16, 8), (13, 7)])
def test_brute_force_tiny(oracle_mod, causal, N, d):
    """Element-by-element agreement with an independent brute force.
    Catches a wrong (b, h) offset (B*H = 4 here), index or sign anywhere."""
    B, H = 2, 2
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=100 + N + d))
    scale = 0.3
    o, lse = oracle_mod.attn_ref(q, k, v, causal, scale)
    Q, K, V = f64(q), f64(k), f64(v)
    for b in range(B):
        for h in range(H):
            ob, lb = _brute_long_double(Q[b, h], K[b, h], V[b, h], causal, scale)
            np.testing.assert_allclose(o[b, h], ob.astype(np.float64), rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], lb.astype(np.float64), rtol=0, atol=1e-13)


def test_row_subset_matches_full(oracle_mod):
    """Computing a listed subset of rows gives the same bits as the full run
    (the row-sampled checks on large workloads rely on this)."""
    B, H, N, d = 2, 2, 50, 16
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=16))
    o, lse = oracle_mod.attn_ref(q, k, v, True, 0.25)
    rows = np.array([0, 7, 49, 50, 99, 150, 199], dtype=np.int64)
    os_, ls_ = oracle_mod.attn_ref(q, k, v, True, 0.25, rows=rows)
    np.testing.assert_array_equal(os_, o.reshape(-1, d)[rows])
    np.testing.assert_array_equal(ls_, lse.reshape(-1)[rows])


def test_rejects_bad_rows(oracle_mod):
    q, k, v = (bf16_bits(t) for t in make_qkv(1, 1, 4, 4, seed=1))
    with pytest.raises(ValueError):
        oracle_mod.attn_ref(q, k, v, False, 1.0, rows=np.array([4]))


# ------------------------------------------------------ algebraic checks ---
def test_linear_in_v(oracle_mod):
    """O(2 V1 - 3 V2) = 2 O(V1) - 3 O(V2) (small integers: bf16-exact)."""
    B, H, N, d = 1, 2, 19, 8
    q, k, _ = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=17))
    rng = np.random.default_rng(0)
    v1 = rng.integers(-4, 5, size=(B, H, N, d)).astype(np.float64)
    v2 = rng.integers(-4, 5, size=(B, H, N, d)).astype(np.float64)
    for causal in (False, True):
        o1, _ = oracle_mod.attn_ref(q, k, to_bits(v1), causal, 0.4)
        o2, _ = oracle_mod.attn_ref(q, k, to_bits(v2), causal, 0.4)
        o3, _ = oracle_mod.attn_ref(q, k, to_bits(2 * v1 - 3 * v2), causal, 0.4)
        np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, rtol=0, atol=1e-12)


def test_joint_key_value_permutation(oracle_mod):
    """Non-causal: permuting K and V rows together changes nothing."""
    B, H, N, d = 1, 1, 21, 16
    q, k, v = (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=18))
    perm = np.random.default_rng(1).permutation(N)
    o, lse = oracle_mod.attn_ref(q, k, v, False, 0.3)
    op, lp = oracle_mod.attn_ref(q, k[:, :, perm].copy(), v[:, :, perm].copy(), False, 0.3)
    np.testing.assert_allclose(op, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lp, lse, rtol=0, atol=1e-13)


def test_constant_score_shift(oracle_mod):
    """Appending coordinate c to every query and 1 to every key adds
    scale*c to each score: LSE moves by scale*c, O does not move."""
    B, H, N, d = 1, 2, 17, 7
    q, k, v = (f64(bits_) for bits_ in (bf16_bits(t) for t in make_qkv(B, H, N, d, seed=19)))
    c, scale = 6.0, 0.5
    q2 = np.concatenate([q, np.full((B, H, N, 1), c)], -1)
    k2 = np.concatenate([k, np.ones((B, H, N, 1))], -1)
    v2 = np.concatenate([v, np.zeros((B, H, N, 1))], -1)
    for causal in (False, True):
        o, lse = oracle_mod.attn_ref(to_bits(q), to_bits(k), to_bits(v), causal, scale)
        o2, lse2 = oracle_mod.attn_ref(to_bits(q2), to_bits(k2), to_bits(v2), causal, scale)
        np.testing.assert_allclose(o2[..., :d], o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse2, lse + scale * c, rtol=0, atol=1e-12)


# ------------------------------------------------- tiled algorithm model ---
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 8.0, 30.0])
def test_tiled_online_model_equals_plain_definition(oracle_mod, causal, tau):
    """The tiled, running-max, lazily rescaled algorithm reaches the plain
    definition (tiling and a conditional rescale only reorder the sum).
    N = 300 spans several 128-wide tiles and a ragged tail; Q ~ 3 N(0,1)
    makes the running maximum jump."""
    N, d = 300, 32
    q, k, v = (bf16_bits(t) for t in make_qkv(1, 1, N, d, seed=20, q_std=3.0))
    scale = 1 / math.sqrt(d)
    o, lse = oracle_mod.attn_ref(q, k, v, causal, scale)
    om, lm = oracle_mod.tiled_online_model(f64(q)[0, 0], f64(k)[0, 0], f64(v)[0, 0], causal,
                                           scale, block_n=128, tau=tau)
    np.testing.assert_allclose(om, o[0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, lse[0, 0], rtol=0, atol=1e-12)


def test_lazy_rescale_keeps_weights_bounded():
    """Under the lazy condition every weight stays <= 2**tau, so the fp32
    running sum and the bf16 weights cannot overflow (section "Deplacer une
    partie des exponentielles": the final normalisation cannot repair an
    overflow).  Checked by replaying the model's maxima on peaky scores."""
    import oracle
    N, d, tau = 512, 64, 8.0
    q, k, v = (f64(bf16_bits(t))[0, 0] for t in make_qkv(1, 1, N, d, seed=21, q_std=3.0))
    scale = 1 / math.sqrt(d)
    x = (q @ k.T) * scale / math.log(2)
    m = np.full(N, -np.inf)
    for j0 in range(0, N, 128):
        t = x[:, j0:j0 + 128]
        new_m = np.maximum(m, t.max(1))
        m = np.where(new_m - m > tau, new_m, m)
        assert (np.exp2(t - m[:, None]) <= 2 ** tau * (1 + 1e-12)).all()
    om, _ = oracle.tiled_online_model(q, k, v, False, scale, tau=tau)
    assert np.isfinite(om).all()


def test_bf16_weight_rounding_error_is_inside_tolerance(oracle_mod):
    """Predicts the kernel's error budget: rounding the weights to bf16
    before the second product moves O by far less than the parity tolerance
    (2e-2 absolute + 1e-2 relative): at most half of it, elementwise."""
    N, d = 1024, 128
    q, k, v = (bf16_bits(t) for t in make_qkv(1, 1, N, d, seed=22, q_std=3.0))
    scale = 1 / math.sqrt(d)
    o, _ = oracle_mod.attn_ref(q, k, v, True, scale)
    om, _ = oracle_mod.tiled_online_model(f64(q)[0, 0], f64(k)[0, 0], f64(v)[0, 0], True, scale,
                                          tau=8.0, round_p_bf16=True)
    err = np.abs(om - o[0, 0])
    # Peaky causal rows put most weight on a few keys, so one weight's bf16
    # rounding (relative 2**-9) shows almost undamped: about 40% of the budget.
    assert (err <= 0.5 * (2e-2 + 1e-2 * np.abs(o[0, 0]))).all()
