"""GPU parity of the CTA-pair kernel (attn_fwd_pair: clusters of two CTAs
sharing each M = 256 tensor-core product) against the fp64 oracle, with the
tolerance of the one-CTA kernel: |O_gpu - O_ref| <= 2e-2 + 1e-2 |O_ref| and
|LSE_gpu - LSE_ref| <= 1e-3."""
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import (WORKLOADS, bf16_bits, make_qkv,
                                                    make_workload_inputs, sample_rows)

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 2e-2, 1e-2, 1e-3


def check(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all(), what
    err_o = np.abs(o_gpu - o_ref)
    bad = err_o > ATOL_O + RTOL_O * np.abs(o_ref)
    assert not bad.any(), f"{what}: {bad.sum()} O elements out of tolerance, max err {err_o.max():.3g}"
    err_l = np.abs(lse_gpu - lse_ref)
    assert err_l.max() <= ATOL_LSE, f"{what}: LSE max err {err_l.max():.3g}"


def pair_run(q, k, v, causal, scale):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = tab.attn_fwd_pair(qd, kd, vd, causal=causal, scale=scale)
    assert tab.last_device_error() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def full_parity(oracle_mod, B, H, N, causal, seed, q_std=1.0, scale=None):
    d = 128
    scale = 1 / math.sqrt(d) if scale is None else scale
    q, k, v = make_qkv(B, H, N, d, seed, q_std)
    o, lse = pair_run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    check(o, lse, o_ref, lse_ref, f"pair B{B} H{H} N{N} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 256, 512, 640, 1024, 1536])
def test_pair_small_shapes(oracle_mod, causal, N):
    """One tile (the other three of the group of four are empty), one full
    group of four tiles, and several groups with K/V tiles that only one
    CTA's rows can see under the mask."""
    full_parity(oracle_mod, 2, 3, N, causal, seed=4000 + N + causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 100, 129, 300, 700])
def test_pair_ragged_lengths(oracle_mod, causal, N):
    """N not a multiple of 128 (nor of 512): the rows of one CTA of a pair
    may lie wholly past the end; keys past N are masked."""
    full_parity(oracle_mod, 2, 3, N, causal, seed=4100 + N, q_std=2.0)


@pytest.mark.parametrize("causal", [False, True])
def test_pair_peaky_scores(oracle_mod, causal):
    full_parity(oracle_mod, 1, 4, 1024, causal, seed=4200, q_std=3.0)


@pytest.mark.parametrize("name", ["b4h16n2048d128_causal"])
def test_pair_workload_full(oracle_mod, name):
    w = WORKLOADS[name]
    full_parity(oracle_mod, w.B, w.H, w.N, w.causal, w.seed, w.q_std)


@pytest.mark.parametrize("name", ["b2h32n8192d128_causal", "b8h16n4096d128_peaky"])
def test_pair_workload_sampled_rows(oracle_mod, name):
    """Full-size workloads; the oracle computes the deterministic row sample
    the one-CTA kernel's tests use."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    o, lse = pair_run(q, k, v, w.causal, w.scale)
    rows = sample_rows(w, n_random=256)
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal,
                                         w.scale, rows=rows)
    check(o.reshape(-1, w.d)[rows], lse.reshape(-1)[rows], o_ref, lse_ref, name)


@pytest.mark.parametrize("causal", [False, True])
def test_pair_every_output_written_and_guards_intact(causal):
    B, H, N, d = 1, 3, 700, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, 4300))
    g = 4096
    o_buf = torch.full((g + B * H * N * d + g,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((g + B * H * N + g,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[g:g + B * H * N * d].view(B, H, N, d)
    lse = l_buf[g:g + B * H * N].view(B, H, N)
    tab.attn_fwd_pair_into(q, k, v, o, lse, causal=causal)
    assert tab.last_device_error() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert torch.isnan(o_buf[:g]).all() and torch.isnan(o_buf[-g:]).all()
    assert torch.isnan(l_buf[:g]).all() and torch.isnan(l_buf[-g:]).all()


def test_pair_deterministic_and_close_to_one_cta_kernel():
    """Bitwise repeatable; within rounding of the one-CTA kernel (the same
    arithmetic, products accumulated in another grouping)."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 2048, 128, 4400))
    o1, l1 = tab.attn_fwd_pair(q, k, v, causal=True)
    for _ in range(3):
        o2, l2 = tab.attn_fwd_pair(q, k, v, causal=True)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o_ref, l_ref = tab.attn_fwd(q, k, v, causal=True)
    assert (o1.float() - o_ref.float()).abs().max().item() <= 2e-2
    assert (l1 - l_ref).abs().max().item() <= 1e-3


def test_pair_rejects_other_head_dims():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tab.AttnError):
        tab.attn_fwd_pair(q, q, q)
