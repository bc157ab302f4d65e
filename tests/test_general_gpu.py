"""GPU parity of the general forms against the fp64 oracle: queries and keys
of different lengths with a causal offset and shared K/V heads
(attn_fwd_chunk), packed variable-length batches (attn_fwd_varlen), key
slices merged by LSE (attn_fwd_splitkv) and the merge itself (attn_combine).

Same tolerance as the square case: |O - O_ref| <= 2e-2 + 1e-2 |O_ref|
elementwise, |LSE - LSE_ref| <= 1e-3; rows that see no key must come out as
O = 0 and LSE = -inf exactly.
"""
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import bf16_bits, make_qkv

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 2e-2, 1e-2, 1e-3


def check(o, lse, o_ref, lse_ref, what):
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: rows with no key differ"
    assert np.isfinite(o).all() and np.isfinite(lse[~empty]).all(), what
    bad = np.abs(o - o_ref) > ATOL_O + RTOL_O * np.abs(o_ref)
    assert not bad.any(), f"{what}: {bad.sum()} O elements out of tolerance, " \
                          f"max err {np.abs(o - o_ref).max():.3g}"
    if (~empty).any():
        err = np.abs(lse[~empty] - lse_ref[~empty]).max()
        assert err <= ATOL_LSE, f"{what}: LSE max err {err:.3g}"


def draw(B, H, H_kv, N_q, N_k, d, seed, q_std=1.0):
    q = make_qkv(B, H, N_q, d, seed, q_std)[0]
    _, k, v = make_qkv(B, H_kv, N_k, d, seed + 7)
    return q, k, v


# ------------------------------------------------------------- chunk ---
@pytest.mark.parametrize("out", ["bf16", "fp32"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,delta", [
    (1, 4, 4, 300, 1000, 128, 700),   # queries are the last 300 of 1000 positions
    (2, 8, 2, 1, 4096, 128, 4095),    # one query per head (decode), 4 query heads per K/V head
    (1, 3, 1, 640, 256, 64, -384),    # more queries than keys: early rows see nothing
    (2, 2, 2, 257, 257, 96, 64),      # diagonal offset by half a tile
    (1, 2, 1, 200, 700, 128, -100),   # negative offset: rows 0..99 see nothing
    (1, 4, 2, 300, 900, 256, 600),    # head dim 256
])
def test_chunk_matches_oracle(oracle_mod, out, causal, B, H, H_kv, N_q, N_k, d, delta):
    scale = 1 / math.sqrt(d)
    q, k, v = draw(B, H, H_kv, N_q, N_k, d, seed=500 + N_q + N_k + d, q_std=2.0)
    o, lse = tab.attn_fwd_chunk(q.cuda(), k.cuda(), v.cuda(), causal, delta, scale,
                                out_dtype=torch.float32 if out == "fp32" else torch.bfloat16)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                               causal, delta, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
          f"chunk B{B} H{H}/{H_kv} Nq{N_q} Nk{N_k} d{d} delta{delta} causal={causal}")


def test_chunk_square_equals_attn_fwd():
    """N_q = N_k, H_kv = H, delta = 0: bit-identical to attn_fwd."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 1000, 128, 61))
    for causal in (False, True):
        o1, l1 = tab.attn_fwd(q, k, v, causal=causal)
        o2, l2 = tab.attn_fwd_chunk(q, k, v, causal, 0)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------ varlen ---
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,H,H_kv,lens_q,lens_k", [
    (128, 4, 2, [300, 0, 1, 1024, 77], [300, 5, 700, 1024, 77]),
    (64, 2, 2, [129, 513, 3], [129, 513, 3]),
    (96, 6, 3, [256, 40], [1000, 0]),
    (256, 2, 1, [700, 130], [700, 900]),
])
def test_varlen_matches_oracle(oracle_mod, causal, d, H, H_kv, lens_q, lens_k):
    scale = 1 / math.sqrt(d)
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    T_q, T_k = int(cu_q[-1]), int(cu_k[-1])
    seed = 700 + T_q + d
    q = make_qkv(1, 1, T_q * H, d, seed, 2.0)[0].reshape(T_q, H, d)
    _, k, v = make_qkv(1, 1, T_k * H_kv, d, seed + 1)
    k = k.reshape(T_k, H_kv, d)
    v = v.reshape(T_k, H_kv, d)
    o, lse = tab.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(),
                                 torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                                 max(lens_q), max(lens_k), causal, scale)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_varlen(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                              cu_q, cu_k, causal, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
          f"varlen d{d} H{H}/{H_kv} q{lens_q} k{lens_k} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_short_query_blocks_pack_heads(oracle_mod, causal):
    """64 sequences of at most 128 queries (some with none) against up to
    800 keys (some with none), 4 query heads per K/V head: two query heads
    share each work item (256 items)."""
    rng = np.random.default_rng(77)
    B, H, H_kv, d = 64, 8, 2, 128
    lens_q = rng.integers(0, 129, B)
    lens_k = rng.integers(0, 801, B)
    lens_q[:3] = [0, 128, 1]
    lens_k[:3] = [10, 0, 800]
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    T_q, T_k = int(cu_q[-1]), int(cu_k[-1])
    q = make_qkv(1, 1, T_q * H, d, 1600, 2.0)[0].reshape(T_q, H, d)
    _, k, v = make_qkv(1, 1, T_k * H_kv, d, 1601)
    k, v = k.reshape(T_k, H_kv, d), v.reshape(T_k, H_kv, d)
    scale = 1 / math.sqrt(d)
    o, lse = tab.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(),
                                 torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                                 int(lens_q.max()), int(lens_k.max()), causal, scale)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_varlen(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                              cu_q, cu_k, causal, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"varlen packed causal={causal}")


def test_varlen_packed_heads_bad_offsets_are_caught():
    """Packed items (200) with one sequence longer than max_seqlen_q: that
    sequence is skipped with ATTN_ERR_DEVICE_BOUNDS, the others computed."""
    B, H, H_kv, d = 100, 4, 2, 128
    lens = np.full(B, 100)
    lens[7] = 150
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)).cuda()
    T = int(lens.sum())
    q = make_qkv(1, 1, T * H, d, 1700)[0].reshape(T, H, d).cuda()
    _, k, v = make_qkv(1, 1, T * H_kv, d, 1701)
    k, v = k.reshape(T, H_kv, d).cuda(), v.reshape(T, H_kv, d).cuda()
    o, lse = tab.attn_fwd_varlen(q, k, v, cu, cu, 128, 200, True)
    assert tab.last_device_error() == -6
    assert tab.last_device_error() == 0
    assert torch.isfinite(o[:700]).all() and torch.isfinite(lse[:, :700]).all()


def test_varlen_bad_offsets_are_caught_on_the_device():
    """A sequence longer than max_seqlen_q is skipped and reported as
    ATTN_ERR_DEVICE_BOUNDS; the other sequences are still computed, and the
    next launch is clean."""
    H, d = 2, 128
    cu = torch.tensor([0, 100, 400], dtype=torch.int32, device="cuda")
    q, k, v = (t.reshape(400, H, d).cuda() for t in make_qkv(1, 1, 400 * H, d, 81))
    o, lse = tab.attn_fwd_varlen(q, k, v, cu, cu, 200, 300, True)
    assert tab.last_device_error() == -6
    assert tab.last_device_error() == 0
    assert torch.isfinite(o[:100]).all() and torch.isfinite(lse[:, :100]).all()


# ----------------------------------------------------------- split-KV ---
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,d,n_splits", [
    (1, 2, 2, 4096, 4096, 128, 8),
    (1, 1, 1, 1000, 1000, 64, 3),
    (2, 1, 1, 2300, 2300, 96, 5),
    (1, 2, 2, 640, 640, 128, 64),   # more slices asked for than tiles: one tile each
    (1, 8, 2, 128, 8192, 128, 16),  # a block of queries against a long cache
    (2, 4, 4, 1, 3000, 128, 7),     # one query per head
    (1, 2, 1, 256, 4096, 256, 6),   # head dim 256
])
def test_splitkv_matches_oracle(oracle_mod, causal, B, H, H_kv, N_q, N_k, d, n_splits):
    scale = 1 / math.sqrt(d)
    delta = N_k - N_q  # the queries are the last N_q positions
    q, k, v = draw(B, H, H_kv, N_q, N_k, d, 900 + N_q + N_k + d, 2.0)
    o, lse = tab.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), n_splits, causal, delta, scale)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal,
                                               delta, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
          f"splitkv B{B} H{H}/{H_kv} Nq{N_q} Nk{N_k} d{d} slices{n_splits} causal={causal}")


# Packed items are used when they number at least 2/3 of the SMs (99 of 148),
# so every case below has 128 or more of them.
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,H_kv,N_q,N_k,n_splits", [
    (2, 6, 2, 128, 3000, 32),  # 3 query heads per K/V head: one item holds a single head
    (1, 8, 2, 100, 2000, 64),  # ragged query block
    (2, 4, 1, 1, 5000, 64),    # decode: one query per head
    (8, 32, 16, 64, 700, 1),   # 2 query heads per K/V head, no key slices
])
def test_query_heads_sharing_kv_are_packed(oracle_mod, causal, B, H, H_kv, N_q, N_k, n_splits):
    """Up to 128 queries per head with K/V heads shared: each work item pairs
    two query heads of one K/V head (one K/V stream, both softmax groups).
    Against the oracle, for full and single-head items and key slices
    (including slices past the last key tile, which see no key)."""
    d = 128
    scale = 1 / math.sqrt(d)
    delta = N_k - N_q
    q, k, v = draw(B, H, H_kv, N_q, N_k, d, 1300 + N_q + N_k + H, 2.0)
    if n_splits == 1:
        o, lse = tab.attn_fwd_chunk(q.cuda(), k.cuda(), v.cuda(), causal, delta, scale)
    else:
        o, lse = tab.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), n_splits, causal, delta, scale)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal,
                                               delta, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref,
          f"packed B{B} H{H}/{H_kv} Nq{N_q} Nk{N_k} slices{n_splits} causal={causal}")


@pytest.mark.parametrize("delta", [-100, 72])
def test_packed_heads_with_rows_that_see_no_key(oracle_mod, delta):
    """Packed items (128 of them) under a causal offset that leaves the first
    rows without a visible key (delta < 0), or shifts the diagonal inside
    the tile: those rows come out as O = 0, LSE = -inf in both heads."""
    B, H, H_kv, N_q, N_k, d = 64, 4, 2, 128, 200, 128
    scale = 1 / math.sqrt(d)
    q, k, v = draw(B, H, H_kv, N_q, N_k, d, 1500 + delta, 2.0)
    o, lse = tab.attn_fwd_chunk(q.cuda(), k.cuda(), v.cuda(), True, delta, scale)
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v), True,
                                               delta, scale)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"packed delta={delta}")


def test_packed_heads_equal_one_head_per_item():
    """Each query head's result does not depend on the head it shares an
    item with: the packed launch (128 items) equals one-head launches
    (unpacked) bitwise."""
    B, H, H_kv, N_q, N_k, d = 64, 4, 2, 128, 1500, 128
    q, k, v = (t.cuda() for t in draw(B, H, H_kv, N_q, N_k, d, 1400))
    o, lse = tab.attn_fwd_chunk(q, k, v, True, N_k - N_q)
    for h in range(H):
        hk = h // (H // H_kv)
        o1, l1 = tab.attn_fwd_chunk(q[:, h:h + 1].contiguous(), k[:, hk:hk + 1].contiguous(),
                                    v[:, hk:hk + 1].contiguous(), True, N_k - N_q)
        assert torch.equal(o[:, h:h + 1], o1) and torch.equal(lse[:, h:h + 1], l1)


def test_splitkv_one_slice_is_attn_fwd():
    q, k, v = (t.cuda() for t in make_qkv(1, 2, 700, 128, 91))
    o1, l1 = tab.attn_fwd(q, k, v, causal=True)
    o2, l2 = tab.attn_fwd_splitkv(q, k, v, 1, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------ combine ---
@pytest.mark.parametrize("d", [64, 96, 128, 256])
def test_combine_matches_oracle_merge(oracle_mod, d):
    """Random parts (with some parts and some whole rows unseen, LSE = -inf)
    merged on the GPU against the oracle's merge."""
    G, rows = 5, 3000
    rng = np.random.default_rng(d)
    o_parts = rng.standard_normal((G, rows, d)).astype(np.float32)
    lse_parts = (rng.standard_normal((G, rows)) * 4).astype(np.float32)
    lse_parts[rng.random((G, rows)) < 0.2] = -np.inf
    lse_parts[:, :7] = -np.inf
    o, lse = tab.attn_combine(torch.from_numpy(o_parts).cuda(), torch.from_numpy(lse_parts).cuda())
    o_ref, l_ref = oracle_mod.lse_merge(o_parts, lse_parts)
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, f"combine d{d}")
    o32, _ = tab.attn_combine(torch.from_numpy(o_parts).cuda(), torch.from_numpy(lse_parts).cuda(),
                              out_dtype=torch.float32)
    np.testing.assert_allclose(o32.cpu().numpy(), o_ref, rtol=1e-5, atol=1e-5)


def test_chunks_over_key_slices_combine_to_the_whole(oracle_mod):
    """The context-parallel recipe on one GPU: each key slice through
    attn_fwd_chunk (fp32 O, causal offset shifted by the slice start), then
    attn_combine, equals the oracle on all keys."""
    B, H, N, d = 1, 4, 1536, 128
    q, k, v = make_qkv(B, H, N, d, 95)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cuts = [0, 384, 1000, 1536]
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o_g, l_g = tab.attn_fwd_chunk(qd, kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous(),
                                      True, -a, out_dtype=torch.float32)
        parts_o.append(o_g)
        parts_l.append(l_g)
    o, lse = tab.attn_combine(torch.stack(parts_o), torch.stack(parts_l))
    assert tab.last_device_error() == 0
    o_ref, l_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), True,
                                       1 / math.sqrt(d))
    check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "chunks + combine")


# ------------------------------------------ measured general workloads ---
@pytest.mark.parametrize("name", sorted(__import__(
    "tiled_attention_forward_sm_b200.inputs", fromlist=["GENERAL_WORKLOADS"]).GENERAL_WORKLOADS))
def test_general_workloads_sampled_parity(oracle_mod, name):
    """The measured general workloads at their full sizes, through the same
    entry points bench.py times, on seeded sampled rows against the oracle."""
    from tiled_attention_forward_sm_b200.inputs import GENERAL_WORKLOADS, make_general_inputs
    w = GENERAL_WORKLOADS[name]
    q, k, v = make_general_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rng = np.random.default_rng(77)
    if w.kind == "varlen":
        cu_q = np.concatenate([[0], np.cumsum(w.lens_q)]).astype(np.int32)
        cu_k = np.concatenate([[0], np.cumsum(w.lens_k)]).astype(np.int32)
        o, lse = tab.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(cu_q).cuda(),
                                     torch.from_numpy(cu_k).cuda(), w.N_q, w.N_k, w.causal, w.scale)
        assert tab.last_device_error() == 0
        o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
        qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
        for b in range(w.B):
            q0, q1, k0, k1 = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
            nq = q1 - q0
            toks = np.unique(np.concatenate([[0, nq - 1], rng.integers(0, nq, 6)]))
            rows = np.concatenate([h * nq + toks for h in range(w.H)]).astype(np.int64)
            o_ref, l_ref = oracle_mod.attn_ref_general(
                qb[q0:q1].transpose(1, 0, 2)[None], kb[k0:k1].transpose(1, 0, 2)[None],
                vb[k0:k1].transpose(1, 0, 2)[None], w.causal, (k1 - k0) - nq, w.scale, rows=rows)
            o_g = np.concatenate([o[q0 + toks, h] for h in range(w.H)])
            l_g = np.concatenate([lse[h, q0 + toks] for h in range(w.H)])
            check(o_g, l_g, o_ref, l_ref, f"{name} sequence {b}")
        return
    delta = w.N_k - w.N_q
    if w.kind == "chunk":
        o, lse = tab.attn_fwd_chunk(qd, kd, vd, w.causal, delta, w.scale)
    else:
        o, lse = tab.attn_fwd_splitkv(qd, kd, vd, w.n_splits, w.causal, delta, w.scale)
    assert tab.last_device_error() == 0
    total = w.B * w.H * w.N_q
    rows = np.unique(np.concatenate([np.arange(0, total, w.N_q), np.arange(w.N_q - 1, total, w.N_q),
                                     rng.integers(0, total, 512)])).astype(np.int64)
    o_ref, l_ref = oracle_mod.attn_ref_general(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal,
                                               delta, w.scale, rows=rows)
    check(o.float().cpu().numpy().reshape(-1, w.d)[rows], lse.cpu().numpy().reshape(-1)[rows],
          o_ref, l_ref, name)
