"""Pins for the k-means assignment oracle (``oracle.kmeans_assign``): closed
forms, invariants and an independent formulation, each named for the
mistake it catches.  The definition (page lefilia.fr, Flash-KMeans item):
every point goes to its nearest centroid."""
import numpy as np
import pytest
import torch

from tiled_attention_forward_sm_b200.inputs import bf16_bits


def bits(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "fixture value not exactly bf16"
    return bf16_bits(b)


def f64(b) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bits(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return bf16_bits(torch.randn(shape, generator=g).to(torch.bfloat16))


def test_points_on_centroids(oracle_mod):
    """A point equal to centroid j is assigned to j at distance exactly 0
    (catches a wrong index or a sign error in the difference)."""
    c = rand_bits((9, 16), 1)
    a, best = oracle_mod.kmeans_assign(c[[4, 0, 8, 4]], c)
    np.testing.assert_array_equal(a, [4, 0, 8, 4])
    np.testing.assert_array_equal(best, 0.0)


def test_one_dimension_closed_form(oracle_mod):
    """d = 1 with sorted centroids: the nearest centroid is found by the
    interval midpoints (small integers and halves: all exact); 0.5 is the
    midpoint of -1 and 2, a tie that goes to the smaller index."""
    cents = np.array([[-6.0], [-1.0], [2.0], [10.0]])
    pts = np.array([[-9.0], [-3.0], [-3.5], [0.0], [0.5], [6.0], [6.5], [40.0]])
    a, best = oracle_mod.kmeans_assign(bits(pts), bits(cents))
    np.testing.assert_array_equal(a, [0, 1, 0, 1, 1, 2, 3, 3])
    np.testing.assert_array_equal(best, [9.0, 4.0, 6.25, 1.0, 2.25, 16.0, 12.25, 900.0])


def test_ties_go_to_the_smaller_index(oracle_mod):
    """Duplicated centroids: the first copy wins."""
    c = rand_bits((6, 8), 2)
    c2 = np.concatenate([c, c[::-1]])
    x = rand_bits((40, 8), 3)
    a, _ = oracle_mod.kmeans_assign(x, c2)
    assert (a < 6).all()


def test_matches_expanded_form_with_a_matmul(oracle_mod):
    """An independent formulation, ||x||^2 - 2 x.c + ||c||^2 through a
    numpy matmul in fp64: same minima (to rounding) and the same index
    wherever the best two distances are not within rounding of each other
    (catches a transposed operand or a dropped term)."""
    x, c = rand_bits((300, 64), 4), rand_bits((97, 64), 5)
    a, best, dist = oracle_mod.kmeans_assign(x, c, with_dist=True)
    X, C = f64(x), f64(c)
    D = (X * X).sum(1)[:, None] - 2.0 * X @ C.T + (C * C).sum(1)[None, :]
    np.testing.assert_allclose(dist, D, rtol=1e-12, atol=1e-10)
    np.testing.assert_allclose(best, D.min(1), rtol=1e-12, atol=1e-10)
    srt = np.sort(D, axis=1)
    clear = srt[:, 1] - srt[:, 0] > 1e-9
    np.testing.assert_array_equal(a[clear], D.argmin(1)[clear])


def test_centroid_permutation_and_translation(oracle_mod):
    """Permuting the centroids permutes the assignment; shifting points and
    centroids by one vector changes nothing (integer data: exact)."""
    rng = np.random.default_rng(6)
    x = rng.integers(-20, 21, size=(200, 5)).astype(np.float64)
    c = rng.integers(-20, 21, size=(13, 5)).astype(np.float64)
    c = np.unique(c, axis=0)
    a, best = oracle_mod.kmeans_assign(bits(x), bits(c))
    perm = rng.permutation(len(c))
    a_p, best_p = oracle_mod.kmeans_assign(bits(x), bits(c[perm]))
    np.testing.assert_array_equal(best_p, best)
    inv = np.argsort(perm)
    same = best_p == best
    # where the nearest centroid is unique the permuted index maps back
    dist = ((x[:, None, :] - c[None, :, :]) ** 2).sum(-1)
    unique = (dist == best[:, None]).sum(1) == 1
    np.testing.assert_array_equal(perm[a_p][unique & same], a[unique & same])
    assert inv.shape == perm.shape
    shift = np.array([3.0, -5.0, 7.0, 1.0, -2.0])
    a_s, best_s = oracle_mod.kmeans_assign(bits(x + shift), bits(c + shift))
    np.testing.assert_array_equal(a_s, a)
    np.testing.assert_array_equal(best_s, best)


def test_row_subset_matches_full(oracle_mod):
    x, c = rand_bits((120, 32), 7), rand_bits((40, 32), 8)
    a, best = oracle_mod.kmeans_assign(x, c)
    rows = np.array([0, 5, 119, 64], dtype=np.int64)
    a_r, best_r = oracle_mod.kmeans_assign(x, c, rows=rows)
    np.testing.assert_array_equal(a_r, a[rows])
    np.testing.assert_array_equal(best_r, best[rows])


def test_rejects_bad_rows(oracle_mod):
    x, c = rand_bits((4, 4), 9), rand_bits((2, 4), 10)
    with pytest.raises(ValueError):
        oracle_mod.kmeans_assign(x, c, rows=np.array([4]))
