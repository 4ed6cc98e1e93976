"""Pins for the fp64 cluster-layout oracle: a hand-derived example, a library routine
(scikit-learn's Lloyd k-means from the same initial centroids), planted clusters,
monotone inertia and the permutation's invariants."""
import json
import os

import numpy as np
import pytest

from oracle import cluster_layout as K


def _planted(C, per, d, seed, spread=5.0, noise=0.1):
    """Interleaved planted clusters: token r belongs to cluster r mod C. With per = N / C
    coprime to C, the evenly spaced initial tokens hit every cluster once."""
    rng = np.random.default_rng(seed)
    ids = np.arange(C * per) % C
    centers = spread * rng.standard_normal((C, d))
    return centers[ids] + noise * rng.standard_normal((C * per, d)), ids


def test_golden_kmeans(golden_dir):
    with open(os.path.join(golden_dir, "kmeans_d2.json")) as f:
        g = json.load(f)
    x = np.array(g["x"], float)
    for case in g["cases"]:
        labels, c = K.kmeans(x, g["C"], case["iters"])
        assert labels.tolist() == case["labels"], case["iters"]
        np.testing.assert_allclose(c, case["centroids"], rtol=0, atol=1e-12)
        perm, offsets = K.group_major_permutation(labels, g["C"])
        assert perm.tolist() == case["perm"] and offsets.tolist() == case["offsets"]


@pytest.mark.parametrize("iters", [1, 3, 6])
def test_kmeans_equals_scikit_learn_lloyd(iters):
    sklearn = pytest.importorskip("sklearn.cluster")
    rng = np.random.default_rng(5)
    # overlapping blobs, so that assignments change over the iterations
    x = rng.standard_normal((600, 6)) + np.repeat(rng.standard_normal((12, 6)) * 1.5, 50, axis=0)
    C = 12
    labels, c = K.kmeans(x, C, iters)
    assert np.bincount(labels, minlength=C).min() > 0   # no empty cluster (library relocates them)
    km = sklearn.KMeans(n_clusters=C, init=K.kmeans_init(x, C), n_init=1, max_iter=iters,
                        algorithm="lloyd", tol=0.0).fit(x)
    assert np.array_equal(km.labels_, labels)
    np.testing.assert_allclose(km.cluster_centers_, c, rtol=0, atol=1e-10)


def test_planted_clusters_are_recovered():
    C, per = 32, 9          # gcd(9, 32) = 1
    x, ids = _planted(C, per, 16, 1)
    labels, c = K.kmeans(x, C, 2)
    # initial centroid m sits on token floor(m N / C) = 9 m, i.e. planted cluster 9 m mod C
    relabel = (np.arange(C) * per) % C
    assert np.array_equal(relabel[labels], ids)
    assert np.all(K.assignment_margins(x, c) > 1.0)


def test_inertia_never_increases():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((800, 8))
    prev = np.inf
    for t in range(8):
        labels, c = K.kmeans(x, 20, t)
        inertia = float(((x - c[labels]) ** 2).sum())
        assert inertia <= prev + 1e-9
        prev = inertia


def test_group_major_permutation_invariants():
    rng = np.random.default_rng(7)
    C = 9
    labels = rng.integers(0, C - 1, size=500)       # cluster C - 1 stays empty
    perm, offsets = K.group_major_permutation(labels, C)
    assert sorted(perm.tolist()) == list(range(500))
    lp = labels[perm]
    assert np.all(np.diff(lp) >= 0)
    for m in range(C):
        seg = perm[offsets[m]:offsets[m + 1]]
        assert np.all(labels[seg] == m) and np.all(np.diff(seg) > 0)   # stable
    assert offsets[-1] == 500 and offsets[C - 1] == offsets[C]
    y = rng.standard_normal((500, 3))
    assert np.array_equal(K.unpermute_rows(K.permute_rows(y, perm), perm), y)
    # an already grouped layout is left as it is
    perm2, _ = K.group_major_permutation(np.sort(labels), C)
    assert np.array_equal(perm2, np.arange(500))


def test_distances_match_the_difference_form():
    rng = np.random.default_rng(8)
    x, c = rng.standard_normal((50, 7)), rng.standard_normal((6, 7))
    want = ((x[:, None, :] - c[None, :, :]) ** 2).sum(-1)
    np.testing.assert_allclose(K.sq_distances(x, c), want, rtol=0, atol=1e-12)
