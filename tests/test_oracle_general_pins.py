"""Pins for the oracle's general forms: N_q queries against N_k keys with a
causal offset and shared K/V heads (``attn_ref_general``), packed
variable-length batches (``attn_ref_varlen``) and the merge of results over
disjoint key sets (``lse_merge``).

Each check goes through something other than the function under test: an
independent long-double brute force, the already pinned ``attn_ref``, closed
forms for empty and fully visible rows, and the identity "attention over a
union of key sets = merge of attention over each set".  Each test names the
mistake it is there to catch.
"""
import numpy as np
import pytest

from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv


def f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _draw(B, H, H_kv, N_q, N_k, d, seed):
    q = bf16_bits(make_qkv(B, H, N_q, d, seed)[0])
    _, k, v = make_qkv(B, H_kv, N_k, d, seed + 7)
    return q, bf16_bits(k), bf16_bits(v)


def _brute(Q, K, V, causal, delta, scale):
    """Plain loops in long double, no max subtraction; visible keys j < N_k
    with j <= i + delta under the mask; an empty row gives O = 0, LSE = -inf."""
    ld = np.longdouble
    N_q, d = Q.shape
    N_k = K.shape[0]
    o = np.zeros((N_q, d), dtype=ld)
    lse = np.zeros(N_q, dtype=ld)
    for i in range(N_q):
        J = [j for j in range(N_k) if (not causal or j <= i + delta)]
        if not J:
            lse[i] = -np.inf
            continue
        e = []
        for j in J:
            s = ld(0)
            for c in range(d):
                s += ld(Q[i, c]) * ld(K[j, c])
            e.append(np.exp(ld(scale) * s))
        tot = sum(e, ld(0))
        for x, j in zip(e, J):
            for c in range(d):
                o[i, c] += x * ld(V[j, c]) / tot
        lse[i] = np.log(tot)
    return o.astype(np.float64), lse.astype(np.float64)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,H_kv,N_q,N_k,delta", [
    (2, 2, 5, 9, 4),      # queries are the last 5 of 9 positions
    (4, 2, 7, 3, -4),     # more queries than keys: the first rows see nothing
    (3, 1, 6, 6, 2),      # one K/V head for three query heads, offset diagonal
    (2, 1, 4, 11, -2),
])
def test_general_matches_brute_force(oracle_mod, causal, H, H_kv, N_q, N_k, delta):
    """Catches a wrong K/V head for a query head, a wrong offset sign, an
    off-by-one at the diagonal, or a wrong treatment of rows with no key."""
    B, d, scale = 2, 5, 0.35
    q, k, v = _draw(B, H, H_kv, N_q, N_k, d, seed=300 + H + N_q + N_k)
    o, lse = oracle_mod.attn_ref_general(q, k, v, causal, delta, scale)
    Q, K, V = f64(q), f64(k), f64(v)
    g = H // H_kv
    for b in range(B):
        for h in range(H):
            ob, lb = _brute(Q[b, h], K[b, h // g], V[b, h // g], causal, delta, scale)
            np.testing.assert_allclose(o[b, h], ob, rtol=0, atol=1e-13)
            np.testing.assert_array_equal(np.isneginf(lse[b, h]), np.isneginf(lb))
            fin = np.isfinite(lb)
            np.testing.assert_allclose(lse[b, h][fin], lb[fin], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_general_reduces_to_square_oracle(oracle_mod, causal):
    """N_q = N_k, H_kv = H, delta = 0 is the pinned square case, bit for bit."""
    q, k, v = _draw(2, 3, 3, 40, 40, 16, seed=41)
    o1, l1 = oracle_mod.attn_ref(q, k, v, causal, 0.25)
    o2, l2 = oracle_mod.attn_ref_general(q, k, v, causal, 0, 0.25)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_general_rows_with_no_key(oracle_mod):
    """Under the mask with delta = -N_q every row sees nothing: O = 0 and
    LSE = -inf exactly (not NaN, not the mean of V); with delta = -5 exactly
    rows 5.. see keys 0..i-5."""
    q, k, v = _draw(1, 2, 2, 8, 5, 4, seed=42)
    o, lse = oracle_mod.attn_ref_general(q, k, v, True, -8, 1.0)
    assert np.all(o == 0.0) and np.all(np.isneginf(lse))
    o, lse = oracle_mod.attn_ref_general(q, k, v, True, -5, 1.0)
    assert np.all(o[:, :, :5] == 0.0) and np.all(np.isneginf(lse[:, :, :5]))
    assert np.all(np.isfinite(lse[:, :, 5:]))
    np.testing.assert_allclose(o[:, :, 5], f64(v)[:, :, 0], rtol=0, atol=1e-15)


def test_general_large_offset_is_unmasked(oracle_mod):
    """delta >= N_k - 1 makes every key visible: the causal result equals
    the unmasked one."""
    q, k, v = _draw(1, 2, 1, 9, 13, 8, seed=43)
    o1, l1 = oracle_mod.attn_ref_general(q, k, v, True, 12, 0.3)
    o2, l2 = oracle_mod.attn_ref_general(q, k, v, False, 0, 0.3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_general_rejects_bad_heads(oracle_mod):
    q, k, v = _draw(1, 3, 2, 4, 4, 4, seed=44)
    with pytest.raises(ValueError):
        oracle_mod.attn_ref_general(q, k, v, False, 0, 1.0)


# ------------------------------------------------------------- lse_merge ---
@pytest.mark.parametrize("causal", [False, True])
def test_merge_of_key_slices_equals_whole(oracle_mod, causal):
    """Attention over all keys = merge of attention over disjoint key slices,
    each slice taken with the offset shifted by its first key.  Catches a
    wrong weight (exp(LSE_g - LSE)), a missing normalisation, a wrong slice
    offset, and a mishandled slice that a row cannot see (LSE_g = -inf)."""
    B, H, N_q, N_k, d, delta, scale = 1, 2, 12, 37, 8, 10, 0.4
    q, k, v = _draw(B, H, H, N_q, N_k, d, seed=45)
    o_all, l_all = oracle_mod.attn_ref_general(q, k, v, causal, delta, scale)
    cuts = [0, 5, 17, 18, 37]
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o_g, l_g = oracle_mod.attn_ref_general(q, k[:, :, a:b].copy(), v[:, :, a:b].copy(),
                                               causal, delta - a, scale)
        parts_o.append(o_g.reshape(-1, d))
        parts_l.append(l_g.reshape(-1))
    if causal:
        assert np.isneginf(np.stack(parts_l)).any()  # some slice unseen by some row
    o_m, l_m = oracle_mod.lse_merge(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(o_m, o_all.reshape(-1, d), rtol=0, atol=1e-13)
    np.testing.assert_allclose(l_m, l_all.reshape(-1), rtol=0, atol=1e-13)


def test_merge_special_cases(oracle_mod):
    """One part is returned unchanged; a part with LSE = -inf has no weight;
    all parts empty give O = 0, LSE = -inf; two equal parts give the same O
    and LSE + log 2."""
    rng = np.random.default_rng(3)
    o1 = rng.standard_normal((1, 6, 4))
    l1 = rng.standard_normal((1, 6))
    o, l = oracle_mod.lse_merge(o1, l1)
    np.testing.assert_allclose(o, o1[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, l1[0], rtol=0, atol=1e-15)
    o2 = np.concatenate([o1, rng.standard_normal((1, 6, 4))])
    l2 = np.concatenate([l1, np.full((1, 6), -np.inf)])
    o, l = oracle_mod.lse_merge(o2, l2)
    np.testing.assert_allclose(o, o1[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, l1[0], rtol=0, atol=1e-15)
    o, l = oracle_mod.lse_merge(o2, np.full((2, 6), -np.inf))
    assert np.all(o == 0.0) and np.all(np.isneginf(l))
    o, l = oracle_mod.lse_merge(np.concatenate([o1, o1]), np.concatenate([l1, l1]))
    np.testing.assert_allclose(o, o1[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(l, l1[0] + np.log(2.0), rtol=0, atol=1e-14)


# ------------------------------------------------------------ attn_ref_varlen ---
def test_varlen_equal_lengths_is_the_dense_layout(oracle_mod):
    """Equal lengths, packed token-major, give the per-head result after the
    layout change [T, H, d] <-> [B, H, N, d] (catches a transposed layout or
    a wrong LSE layout)."""
    B, H, H_kv, N_q, N_k, d = 3, 4, 2, 10, 14, 8
    q, k, v = _draw(B, H, H_kv, N_q, N_k, d, seed=46)
    for causal in (False, True):
        o, lse = oracle_mod.attn_ref_general(q, k, v, causal, N_k - N_q, 0.3)
        qp = q.transpose(0, 2, 1, 3).reshape(B * N_q, H, d)
        kp = k.transpose(0, 2, 1, 3).reshape(B * N_k, H_kv, d)
        vp = v.transpose(0, 2, 1, 3).reshape(B * N_k, H_kv, d)
        cu_q = np.arange(B + 1) * N_q
        cu_k = np.arange(B + 1) * N_k
        ov, lv = oracle_mod.attn_ref_varlen(qp, kp, vp, cu_q, cu_k, causal, 0.3)
        np.testing.assert_array_equal(ov, o.transpose(0, 2, 1, 3).reshape(B * N_q, H, d))
        np.testing.assert_array_equal(lv, lse.transpose(1, 0, 2).reshape(H, B * N_q))


def test_varlen_sequences_are_independent(oracle_mod):
    """Each sequence sees only its own keys (catches an offset that lets a
    sequence read its neighbour), the last query of a sequence sees every
    key of it, and a sequence with no keys gives O = 0, LSE = -inf."""
    H, d, scale = 2, 4, 0.5
    lq = [3, 0, 5, 2]
    lk = [4, 2, 5, 0]
    cu_q = np.concatenate([[0], np.cumsum(lq)])
    cu_k = np.concatenate([[0], np.cumsum(lk)])
    q = bf16_bits(make_qkv(1, 1, int(cu_q[-1]) * H, d, 47)[0]).reshape(-1, H, d)
    _, k, v = make_qkv(1, 1, int(cu_k[-1]) * H, d, 48)
    k = bf16_bits(k).reshape(-1, H, d)
    v = bf16_bits(v).reshape(-1, H, d)
    o, lse = oracle_mod.attn_ref_varlen(q, k, v, cu_q, cu_k, True, scale)
    Q, K, V = f64(q), f64(k), f64(v)
    for b in range(len(lq)):
        for h in range(H):
            for i in range(lq[b]):
                t = cu_q[b] + i
                if lk[b] == 0:
                    assert np.all(o[t, h] == 0.0) and np.isneginf(lse[h, t])
                    continue
                Kb = K[cu_k[b]:cu_k[b + 1], h]
                Vb = V[cu_k[b]:cu_k[b + 1], h]
                ob, lb = _brute(Q[t:t + 1, h], Kb, Vb, True, i + lk[b] - lq[b], scale)
                np.testing.assert_allclose(o[t, h], ob[0], rtol=0, atol=1e-13)
                np.testing.assert_allclose(lse[h, t], lb[0], rtol=0, atol=1e-13)
        if lq[b] and lk[b]:
            t_last = cu_q[b + 1] - 1
            full, _ = _brute(Q[t_last:t_last + 1, 0], K[cu_k[b]:cu_k[b + 1], 0],
                             V[cu_k[b]:cu_k[b + 1], 0], False, 0, scale)
            np.testing.assert_allclose(o[t_last, 0], full[0], rtol=0, atol=1e-13)


# ------------------------------------------------------------- FP8 (E4M3) ---
def test_e4m3_decode_matches_torch_for_every_code(oracle_mod):
    """The oracle's E4M3 decoding from the format's definition equals
    torch's float8_e4m3fn for all 256 codes (NaN codes included)."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle_mod.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(mine[ok], ref[ok])


def test_e4m3_rounding_matches_torch_and_saturates(oracle_mod):
    """Round to nearest even over 20 binades (subnormals included) equals
    torch's cast; values past 448 saturate (the kernel's satfinite)."""
    import torch
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200000) * np.exp2(rng.uniform(-14, 8, 200000))
    x = np.clip(x, -447.0, 447.0)
    ref = torch.from_numpy(x).float().to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle_mod.round_e4m3(x), ref)
    np.testing.assert_array_equal(oracle_mod.round_e4m3(np.array([500.0, -1e6, 448.0])),
                                  [448.0, -448.0, 448.0])
    # exact halfway cases go to the even neighbour
    np.testing.assert_array_equal(oracle_mod.round_e4m3(np.array([1.0625, 1.1875, 2.0 ** -10])),
                                  [1.0, 1.25, 0.0])


def test_model_with_e4m3_weights_stays_inside_its_bound(oracle_mod):
    """The tiled model with weights rounded to E4M3 differs from the exact
    result by at most sum_j max(2^-4 w_j, min(w_j, 2^-10 w_max)) |v_j| per
    output element (w the exact normalised weights, w_max the row's
    largest): a weight in E4M3's normal range (>= 2^-6 of the running scale
    2^m) moves by at most 2^-4 of itself, a smaller one by at most the half
    spacing 2^-10 (or itself, when it rounds to zero); the lazy rule keeps m
    at or below the row's true maximum, so the running sum is at least
    1 / w_max and the second term, normalised, is at most 2^-10 w_max.  This
    is the bound the GPU test applies to the kernel; here it is checked on
    the model, with ordinary and peaky scores."""
    from tiled_attention_forward_sm_b200.inputs import make_qkv
    import torch
    def e4(t):
        return t[0, 0].float().to(torch.float8_e4m3fn).double().numpy()
    for q_std, seed in ((1.0, 5), (3.0, 6)):
        q, k, v = make_qkv(1, 1, 1024, 128, seed, q_std)
        Q, K, V = e4(q), e4(k), e4(v)
        scale = 128 ** -0.5
        for causal in (False, True):
            o_ex, _ = oracle_mod.tiled_online_model(Q, K, V, causal, scale)
            o_m, _ = oracle_mod.tiled_online_model(Q, K, V, causal, scale, round_p="e4m3")
            S = Q @ K.T * scale
            if causal:
                S = np.where(np.tril(np.ones_like(S)) > 0, S, -np.inf)
            W = np.exp(S - S.max(1, keepdims=True))
            W /= W.sum(1, keepdims=True)
            dW = np.maximum(2.0 ** -4 * W, np.minimum(W, 2.0 ** -10 * W.max(1, keepdims=True)))
            bound = dW @ np.abs(V)
            err = np.abs(o_m - o_ex)
            assert (err <= bound * (1 + 1e-9) + 1e-12).all()
            # and the bound is not vacuous: the rounding uses a visible part of it
            assert (err / np.maximum(bound, 1e-30)).max() > 0.1


def test_e4m3_encoding_round_trips_every_code(oracle_mod):
    """Encoding the decoded value of every finite code gives the code back
    (both zeros and the subnormals included)."""
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle_mod.e4m3_bits_to_f64(codes)
    ok = ~np.isnan(vals)
    np.testing.assert_array_equal(oracle_mod.e4m3_encode(vals[ok]), codes[ok])


def test_quantize_matches_torch_cast(oracle_mod):
    """bf16 * 2^k -> E4M3 codes equal torch's cast of the same products
    (in range: torch's cast does not saturate)."""
    import torch
    x = torch.randn(50000, generator=torch.Generator().manual_seed(3)).bfloat16()
    for inv in (1.0, 4.0, 0.125):
        q = oracle_mod.quantize_e4m3(bf16_bits(x), inv)
        ref = (x.float() * inv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        np.testing.assert_array_equal(q, ref)
