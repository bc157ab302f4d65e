"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded bf16 inputs.

Tolerance (bf16 I/O, fp32 accumulation): |O_gpu - O_ref| <= 2e-2 + 1e-2 |O_ref|
elementwise and |LSE_gpu - LSE_ref| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import (WORKLOADS, bf16_bits, make_jump_qkv, make_qkv,
                                                    make_workload_inputs, sample_rows)

pytestmark = pytest.mark.gpu

ATOL_O, RTOL_O, ATOL_LSE = 2e-2, 1e-2, 1e-3


def gpu_run(q, k, v, causal, scale, poly=None, stages=None):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = tab.attn_fwd(qd, kd, vd, causal=causal, scale=scale, exp2_poly_pairs=poly,
                          kv_stages=stages)
    assert tab.last_device_error() == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all(), what
    err_o = np.abs(o_gpu - o_ref)
    bad = err_o > ATOL_O + RTOL_O * np.abs(o_ref)
    assert not bad.any(), f"{what}: {bad.sum()} O elements out of tolerance, max err {err_o.max():.3g}"
    err_l = np.abs(lse_gpu - lse_ref)
    assert err_l.max() <= ATOL_LSE, f"{what}: LSE max err {err_l.max():.3g}"
    return err_o.max(), err_l.max()


def full_parity(oracle_mod, B, H, N, d, causal, seed, q_std=1.0, scale=None, poly=None,
                stages=None):
    scale = 1 / math.sqrt(d) if scale is None else scale
    q, k, v = make_qkv(B, H, N, d, seed, q_std)
    o, lse = gpu_run(q, k, v, causal, scale, poly, stages)
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    return check(o, lse, o_ref, lse_ref, f"B{B} H{H} N{N} d{d} causal={causal}")


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 256, 384, 640])
def test_small_shapes(oracle_mod, d, causal, N):
    """Single tile, one pair, an odd number of 128-row tiles (a CTA with one
    Q tile), several K/V tiles with a ragged pair count."""
    full_parity(oracle_mod, 2, 3, N, d, causal, seed=N + d + causal)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 100, 129, 255, 300, 1000])
def test_ragged_lengths(oracle_mod, d, causal, N):
    """N not a multiple of 128: the last K/V tile is masked past N and the
    rows past N are neither computed into nor written."""
    full_parity(oracle_mod, 2, 3, N, d, causal, seed=900 + N + d, q_std=2.0)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_length_writes_nothing_past_the_rows(causal, d):
    """B*H heads of N = 200 rows, packed back to back inside guard bands: no
    head's last, partial tile writes into the next head or past the end (at
    d = 96 no row writes past its 96 columns either)."""
    B, H, N = 1, 3, 200
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, 11))
    g = 4096
    o_buf = torch.full((g + B * H * N * d + g,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((g + B * H * N + g,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[g:g + B * H * N * d].view(B, H, N, d)
    lse = l_buf[g:g + B * H * N].view(B, H, N)
    tab.attn_fwd_into(q, k, v, o, lse, causal=causal)
    assert tab.last_device_error() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert torch.isnan(o_buf[:g]).all() and torch.isnan(o_buf[-g:]).all()
    assert torch.isnan(l_buf[:g]).all() and torch.isnan(l_buf[-g:]).all()


@pytest.mark.parametrize("poly", [0, 1, 2])
@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_exp2_split_variants(oracle_mod, poly, d, causal):
    """Every split of the exponentials between the special-function unit and
    the FMA polynomial meets the same tolerance (peaky scores, masked tiles)."""
    full_parity(oracle_mod, 1, 3, 640, d, causal, seed=31 + poly, q_std=3.0, poly=poly)


@pytest.mark.parametrize("stages", [2, 3, 4, 5])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [200, 1000])
def test_kv_ring_depths(oracle_mod, stages, causal, N):
    """Every depth of the K/V ring (page lecompute.fr/en/kernel-perf/flapping-
    airplanes-thunderkittens-megakernels, section "Prepare the next operation
    without overwriting the current one": a stage is refilled only after its
    last reader is done) gives the oracle's result; a ring of 2 stages holds
    exactly one K and one V tile, so every refill waits on the previous
    step's release.  Ragged lengths, several work items per CTA."""
    full_parity(oracle_mod, 2, 5, N, 128, causal, seed=60 + stages + N, q_std=2.0, stages=stages)


def test_kv_ring_depths_are_bitwise_equal():
    """The ring depth changes when tiles arrive, not what is computed."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 1024, 128, 61))
    o4, l4 = tab.attn_fwd(q, k, v, causal=True)
    for st in (2, 3, 5):
        o, l = tab.attn_fwd(q, k, v, causal=True, kv_stages=st)
        assert torch.equal(o, o4) and torch.equal(l, l4)


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("N", [1, 33, 161, 1000])
def test_store_paths_are_bitwise_equal(d, N):
    """Without the causal mask O leaves through per-warp shared-memory boxes
    and TMA stores by default, and through per-row stores with the 5-stage
    ring (no room for the boxes; d = 128) or as fp32: the same values, last
    tiles whose warps hold no row, some rows or all rows included."""
    q, k, v = (t.cuda() for t in make_qkv(2, 3, N, d, 62 + N + d))
    o, lse = tab.attn_fwd(q, k, v, causal=False)
    assert tab.last_device_error() == 0
    if d == 128:
        o5, l5 = tab.attn_fwd(q, k, v, causal=False, kv_stages=5)
        assert torch.equal(o, o5) and torch.equal(lse, l5)
    o32, l32 = tab.attn_fwd_chunk(q, k, v, causal=False, out_dtype=torch.float32)
    assert torch.equal(lse, l32)
    assert torch.equal(o, o32.to(torch.bfloat16))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 33, 161, 1000])
def test_wide_store_paths_are_bitwise_equal(causal, N):
    """d = 256: bf16 O always leaves through two staging boxes per warp and
    TMA stores (a box rewritten once the store two boxes back has read it);
    fp32 O through per-row stores.  Same values."""
    q, k, v = (t.cuda() for t in make_qkv(2, 3, N, 256, 63 + N))
    o, lse = tab.attn_fwd(q, k, v, causal=causal)
    assert tab.last_device_error() == 0
    o32, l32 = tab.attn_fwd_chunk(q, k, v, causal=causal, out_dtype=torch.float32)
    assert torch.equal(lse, l32)
    assert torch.equal(o, o32.to(torch.bfloat16))


@pytest.mark.parametrize("name", ["b1h2n256d64", "b4h16n2048d128_causal"])
def test_workload_full(oracle_mod, name):
    w = WORKLOADS[name]
    full_parity(oracle_mod, w.B, w.H, w.N, w.d, w.causal, w.seed, w.q_std)


@pytest.mark.parametrize("causal", [False, True])
def test_peaky_scores_exercise_lazy_rescale(oracle_mod, causal):
    """Q ~ 3 N(0,1): the running maximum jumps often; several K/V tiles."""
    full_parity(oracle_mod, 1, 4, 1024, 128, causal, seed=77, q_std=3.0)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("jump_tile,second", [(1, False), (2, True)])
def test_lazy_rescale_at_known_rows(oracle_mod, d, causal, jump_tile, second):
    """Constructed scores (inputs.make_jump_qkv, checked on the CPU by
    tests/test_rescale_inputs.py): at a known K/V tile the running maximum of
    known rows, in both Q tiles of a work item and mixed inside warps, jumps
    by the default threshold + 2 (the rescale is taken), by the threshold
    - 0.5 (just under it: weights that large kept unrescaled) or not at all;
    with ``second`` a further jump at the next tile rescales again.  Scale
    ln 2 makes the raw scores log2 units.  Every element against the oracle."""
    B, H, N = 1, 2, 640
    scale = math.log(2.0)
    q, k, v = make_jump_qkv(B, H, N, d, jump_tile, second, seed=400 + d + jump_tile)
    o, lse = gpu_run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    check(o, lse, o_ref, lse_ref, f"jump at tile {jump_tile} d{d} causal={causal}")


@pytest.mark.parametrize("tau", [0.0, 4.0, 16.0])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_rescale_thresholds(oracle_mod, tau, d, causal):
    """Any lazy-rescale threshold gives the oracle's result (0: an eager
    rescale whenever the maximum grows; 16: weights up to 2^16 kept
    unrescaled), on the constructed jumps and on peaky random scores."""
    B, H, N = 1, 2, 640
    scale = math.log(2.0)
    q, k, v = make_jump_qkv(B, H, N, d, 2, True, seed=450 + d)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = tab.attn_fwd(qd, kd, vd, causal=causal, scale=scale, rescale_tau=tau)
    assert tab.last_device_error() == 0
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
    check(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
          o_ref, lse_ref, f"tau {tau}")
    q, k, v = make_qkv(1, 3, 640, d, 470 + d, q_std=3.0)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o, lse = tab.attn_fwd(qd, kd, vd, causal=causal, rescale_tau=tau)
    assert tab.last_device_error() == 0
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal,
                                         1 / math.sqrt(d))
    check(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
          o_ref, lse_ref, f"tau {tau} peaky")


@pytest.mark.parametrize("scale", [0.01, 0.5, 2.0])
def test_other_scales(oracle_mod, scale):
    full_parity(oracle_mod, 1, 2, 512, 128, True, seed=5, scale=scale)


def test_large_magnitude_scores(oracle_mod):
    """Scores spanning ~+-200 (log2 units): weights underflow to exactly 0
    for all but a few keys; no overflow, LSE still exact."""
    full_parity(oracle_mod, 1, 2, 512, 64, False, seed=6, q_std=8.0, scale=0.5)


@pytest.mark.parametrize("name", ["b2h32n8192d128_causal", "b8h16n4096d128_peaky",
                                  "b1h16n32768d128_causal"])
def test_workload_sampled_rows(oracle_mod, name):
    """Full-size workloads in the launch configuration the benchmark uses;
    the oracle computes a deterministic row sample (first/last 128 rows of
    every head, both rows at every 4th tile boundary, 256 random rows).  At
    N = 32768 the whole sample too: the mid-sequence tiles are where the
    work queue's order decides which CTA owns a pair."""
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w)
    o, lse = gpu_run(q, k, v, w.causal, w.scale)
    rows = sample_rows(w, n_random=256)
    o_ref, lse_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), w.causal,
                                         w.scale, rows=rows)
    check(o.reshape(-1, w.d)[rows], lse.reshape(-1)[rows], o_ref, lse_ref, name)


def test_deterministic_bitwise():
    """No atomics touch the results: 20 launches give the same bits (the
    work queue hands items to different CTAs from run to run)."""
    q, k, v = (t.cuda() for t in make_qkv(2, 4, 1024, 128, 9))
    o1, l1 = tab.attn_fwd(q, k, v, causal=True)
    for _ in range(20):
        o2, l2 = tab.attn_fwd(q, k, v, causal=True)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
def test_every_output_written_and_guards_intact(causal):
    """O and LSE pre-filled with NaN inside guard bands: every element is
    written and no guard byte changes."""
    B, H, N, d = 1, 3, 384, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, 10))
    g = 4096
    o_buf = torch.full((g + B * H * N * d + g,), float("nan"), dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((g + B * H * N + g,), float("nan"), dtype=torch.float32, device="cuda")
    o = o_buf[g:g + B * H * N * d].view(B, H, N, d)
    lse = l_buf[g:g + B * H * N].view(B, H, N)
    tab.attn_fwd_into(q, k, v, o, lse, causal=causal)
    assert tab.last_device_error() == 0
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert torch.isnan(o_buf[:g]).all() and torch.isnan(o_buf[-g:]).all()
    assert torch.isnan(l_buf[:g]).all() and torch.isnan(l_buf[-g:]).all()


def test_host_entry_point_matches_device_entry_point():
    B, H, N, d = 1, 2, 512, 128
    q, k, v = make_qkv(B, H, N, d, 12)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_ref, l_ref = tab.attn_fwd(qd, kd, vd, causal=True)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    od = torch.empty_like(qd); ld = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    tab.attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=True)
    assert torch.equal(oh, o_ref.cpu()) and torch.equal(lh, l_ref.cpu())


@pytest.mark.parametrize("causal", [False, True])
def test_host_entry_point_pipelined_over_head_groups(causal):
    """96 MiB of inputs: the host entry point runs as a pipeline over 8
    groups of 4 heads; every head's result is bitwise that of the device
    entry point on the whole tensor."""
    B, H, N, d = 2, 16, 4096, 128
    q, k, v = make_qkv(B, H, N, d, 13)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o_ref, l_ref = tab.attn_fwd(qd, kd, vd, causal=causal)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.full_like(qh, float("nan")).pin_memory()
    lh = torch.full((B, H, N), float("nan"), dtype=torch.float32).pin_memory()
    od = torch.empty_like(qd); ld = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    tab.attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, causal=causal)
    assert torch.equal(oh, o_ref.cpu()) and torch.equal(lh, l_ref.cpu())


def test_rejected_arguments_launch_nothing():
    q = torch.zeros(1, 1, 128, 80, dtype=torch.bfloat16, device="cuda")  # d = 80: unsupported
    with pytest.raises(tab.AttnError) as e:
        tab.attn_fwd(q, q, q)
    assert e.value.status == -2
    assert tab.last_device_error() == 0


def test_bounded_wait_reports_timeout_and_context_stays_usable(oracle_mod):
    """A wait on a barrier that nothing completes gives up after its limit,
    the status word reports the timeout, and the next launch is correct."""
    tab.selftest_wait_timeout(20000)  # 20 ms
    assert tab.last_device_error() == -5
    assert tab.last_device_error() == 0  # read-and-clear
    full_parity(oracle_mod, 1, 2, 256, 128, True, seed=3)


def test_buffers_not_on_the_device_are_refused_before_launch():
    """Host memory (pinned, which CUDA can see) passed where a device buffer
    belongs: every entry point refuses it with ATTN_ERR_INVALID_ARG before
    encoding a tensor map, so no kernel reads it."""
    import ctypes
    B, H, N, d = 1, 2, 256, 128
    q, k, v = (t.cuda() for t in make_qkv(B, H, N, d, 14))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    host = torch.zeros_like(q.cpu()).pin_memory()
    lib = tab.library()
    s = torch.cuda.current_stream().cuda_stream
    args = (B, H, N, d, 1, ctypes.c_float(0.1), s)
    assert lib.attn_fwd(host.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                        lse.data_ptr(), *args) == -1
    assert lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), host.data_ptr(),
                        lse.data_ptr(), *args) == -1
    assert lib.attn_fwd_pair(q.data_ptr(), host.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), *args) == -1
    assert lib.attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), host.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), *args) == -1
    assert tab.last_device_error() == 0
    # and the same buffers on the device still work
    tab.attn_fwd_into(q, k, v, o, lse, causal=True)
    assert tab.last_device_error() == 0 and torch.isfinite(o).all()


def test_tensor_map_cache_follows_the_buffers(oracle_mod):
    """Launches reuse cached tensor maps keyed by address and shape: the same
    address with a new shape, new contents at a cached address, and calls
    after attn_release all give the oracle's results."""
    causal, d = True, 128
    scale = 1 / math.sqrt(d)
    big = torch.empty(3 * 2 * 4 * 512 * d, dtype=torch.bfloat16, device="cuda")
    for (B, H, N, seed) in ((2, 4, 512, 21), (1, 4, 512, 22), (2, 2, 1024, 23), (2, 4, 512, 24)):
        q, k, v = make_qkv(B, H, N, d, seed)
        n = B * H * N * d
        qd, kd, vd = (big[i * n:(i + 1) * n].view(B, H, N, d) for i in range(3))
        for dst, src in ((qd, q), (kd, k), (vd, v)):
            dst.copy_(src)
        o, lse = tab.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
        assert tab.last_device_error() == 0
        o_ref, l_ref = oracle_mod.attn_ref(bf16_bits(q), bf16_bits(k), bf16_bits(v), causal, scale)
        check(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
              o_ref, l_ref, f"cache B{B} H{H} N{N}")
        if seed == 23:
            assert tab.library().attn_release() == 0
