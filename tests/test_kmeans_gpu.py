"""GPU parity of the k-means assignment kernel against the fp64 oracle.

The kernel forms ||c||^2 - 2 x.c in fp32 from bf16 inputs.  The check per
point: the chosen centroid's exact (fp64) distance is within eps of the
minimum, with eps = 2^-12 (||x||^2 + max_j ||c_j||^2), far above fp32
rounding of a 128-term dot product and far below the distance gap a wrong
index, tile offset or norm would cause; where the exact best two distances
are more than 2 eps apart the index must be the oracle's exactly, and the
reported distance must be within eps of the oracle's.
"""
import numpy as np
import pytest
import torch

import tiled_attention_forward_sm_b200 as tab
from tiled_attention_forward_sm_b200.inputs import bf16_bits

pytestmark = pytest.mark.gpu


def draw(N, K, d, seed):
    g = torch.Generator().manual_seed(seed)
    # points around the centroids, so nearest-centroid gaps vary
    c = torch.randn((K, d), generator=g)
    pick = torch.randint(0, K, (N,), generator=g)
    x = c[pick] + 0.5 * torch.randn((N, d), generator=g)
    return x.to(torch.bfloat16), c.to(torch.bfloat16)


def check(oracle_mod, x, c, assign, best, rows=None):
    xb, cb = bf16_bits(x), bf16_bits(c)
    a_ref, b_ref, dist = oracle_mod.kmeans_assign(xb, cb, rows=rows, with_dist=True)
    X = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    C = (cb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    idx = np.arange(len(X)) if rows is None else rows
    eps = 2.0 ** -12 * ((X[idx] ** 2).sum(1) + (C ** 2).sum(1).max())
    a = assign.cpu().numpy()[idx]
    assert a.min() >= 0 and a.max() < len(C)
    chosen = dist[np.arange(len(idx)), a]
    assert (chosen - b_ref <= eps).all(), "a chosen centroid is not (nearly) the nearest"
    srt = np.sort(dist, axis=1)
    clear = srt[:, 1] - srt[:, 0] > 2 * eps if dist.shape[1] > 1 else np.ones(len(idx), bool)
    np.testing.assert_array_equal(a[clear], a_ref[clear])
    if best is not None:
        assert (np.abs(best.cpu().numpy()[idx].astype(np.float64) - b_ref) <= eps).all()
    return clear.mean()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,K", [(1, 1), (100, 7), (256, 128), (300, 129), (1000, 1000),
                                 (4097, 300)])
def test_assign_matches_oracle(oracle_mod, N, K, d):
    """Single tiles, ragged point and centroid counts, several tiles of each."""
    x, c = draw(N, K, d, seed=N + K + d)
    assign, best = tab.kmeans_assign(x.cuda(), c.cuda())
    assert tab.last_device_error() == 0
    frac = check(oracle_mod, x, c, assign, best)
    assert frac > 0.9


def test_assign_without_best_and_points_on_centroids(oracle_mod):
    """Points equal to centroids pick them (distance 0 is exact in fp32),
    and best may be omitted."""
    _, c = draw(1, 300, 128, seed=5)
    perm = torch.randperm(300, generator=torch.Generator().manual_seed(1))
    x = c[perm]
    assign, best = tab.kmeans_assign(x.cuda(), c.cuda(), with_best=False)
    assert best is None and tab.last_device_error() == 0
    assert torch.equal(assign.cpu().long(), perm)


def test_assign_page_workload_sampled(oracle_mod):
    """The workload the page quotes (N = 65536 points, K = 1024 centroids,
    d = 128), on seeded sampled points."""
    from tiled_attention_forward_sm_b200.inputs import KMEANS_WORKLOADS, make_kmeans_inputs
    w = KMEANS_WORKLOADS["kmeans_n65536_k1024_d128"]
    x, c = make_kmeans_inputs(w)
    assign, best = tab.kmeans_assign(x.cuda(), c.cuda())
    assert tab.last_device_error() == 0
    rows = np.unique(np.concatenate([[0, w.N - 1],
                                     np.random.default_rng(3).integers(0, w.N, 2000)]))
    check(oracle_mod, x, c, assign, best, rows=rows.astype(np.int64))


def test_assign_is_deterministic():
    x, c = draw(5000, 700, 128, seed=9)
    a1, b1 = tab.kmeans_assign(x.cuda(), c.cuda())
    for _ in range(3):
        a2, b2 = tab.kmeans_assign(x.cuda(), c.cuda())
        assert torch.equal(a1, a2) and torch.equal(b1, b2)


@pytest.mark.parametrize("d", [64, 128])
def test_assign_many_points_uses_the_norm_prologue(oracle_mod, d):
    """Enough points for more than four rounds of work items over the SMs
    (the point norms then come from a prologue launch rather than from the
    assignment kernel): the same checks on sampled points, and the
    distances agree with the in-kernel norms of the first points."""
    N, K = 200_000, 300
    x, c = draw(N, K, d, seed=11)
    assign, best = tab.kmeans_assign(x.cuda(), c.cuda())
    assert tab.last_device_error() == 0
    rows = np.unique(np.concatenate([[0, N - 1],
                                     np.random.default_rng(4).integers(0, N, 3000)]))
    check(oracle_mod, x, c, assign, best, rows=rows.astype(np.int64))
    a_small, b_small = tab.kmeans_assign(x[:5000].cuda(), c.cuda())
    assert torch.equal(a_small, assign[:5000])
    np.testing.assert_allclose(b_small.cpu().numpy(), best[:5000].cpu().numpy(),
                               rtol=1e-5, atol=1e-4)
