"""fp64 CPU oracle for the cluster-permuted token layout.

TEST INFRASTRUCTURE ONLY, like ``block_sparse_attention``: only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it; the library never does.

Sources (page title, section):
  [EAR]    "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video Generation
           via Error-aware Routing", §2 A (query and key tokens are first grouped into
           semantic clusters by k-means, so that tokens inside a cluster are similar).
  [SPARSE] "Partition the Support, Reconstruct the Residual: Training-Free Sparse
           Attention for Video Generation and World Models" (SparsePR), §2 C (tokens are
           permuted into contiguous group-major layouts before the block-sparse
           attention runs).

Readings where the pages are silent (each is listed with its reason in the design
notes):
  * k-means is Lloyd's iteration on the rows of one head's Q or K (bf16 values taken
    exactly in fp64), squared Euclidean distance, C clusters, T update steps;
  * the initial centroids are the tokens at indices floor(m N / C), m = 0..C-1;
  * an iteration assigns every token to its nearest centroid (ties to the lowest
    index) and replaces every centroid by the mean of its members; a centroid with no
    member keeps its position; after the T updates the tokens are assigned once more,
    to the final centroids, and that assignment is the result;
  * the layout is group-major and stable: tokens ordered by cluster index, and by their
    original index inside a cluster; blocks of b tokens are then cut from that order
    as from the original one (the last block may be partial);
  * Q and K are clustered separately (C clusters each); V follows K's permutation, and
    the attention output rows are returned to the original query order.
"""
from __future__ import annotations

import numpy as np


def kmeans_init(x: np.ndarray, C: int) -> np.ndarray:
    """Initial centroids: the tokens at evenly spaced indices floor(m N / C)."""
    x = np.asarray(x, np.float64)
    N = x.shape[0]
    return x[(np.arange(C) * N) // C].copy()


def sq_distances(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """||x_r - c_m||^2 for every token r and centroid m, [N, C], in fp64."""
    x = np.asarray(x, np.float64)
    c = np.asarray(c, np.float64)
    return (x * x).sum(1)[:, None] - 2.0 * (x @ c.T) + (c * c).sum(1)[None, :]


def kmeans_assign(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Nearest centroid of every token; ties go to the lowest centroid index."""
    return np.argmin(sq_distances(x, c), axis=1)


def kmeans_update(x: np.ndarray, labels: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Each centroid moved to the mean of its members; one with none stays put."""
    x = np.asarray(x, np.float64)
    out = np.array(c, np.float64, copy=True)
    C = out.shape[0]
    counts = np.bincount(labels, minlength=C)
    sums = np.zeros_like(out)
    np.add.at(sums, labels, x)
    live = counts > 0
    out[live] = sums[live] / counts[live, None]
    return out


def kmeans(x: np.ndarray, C: int, iters: int):
    """Lloyd's k-means from :func:`kmeans_init`: ``iters`` update steps, then the final
    assignment. Returns (labels [N], centroids [C, d])."""
    c = kmeans_init(x, C)
    for _ in range(iters):
        c = kmeans_update(x, kmeans_assign(x, c), c)
    return kmeans_assign(x, c), c


def assignment_margins(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """Gap between the second-nearest and the nearest centroid of every token."""
    d = np.sort(sq_distances(x, c), axis=1)
    return d[:, 1] - d[:, 0] if d.shape[1] > 1 else np.full(d.shape[0], np.inf)


def group_major_permutation(labels: np.ndarray, C: int):
    """Stable group-major order: perm[p] = the original index of the token at position
    p; offsets[m] .. offsets[m+1] are the positions of cluster m."""
    labels = np.asarray(labels)
    perm = np.argsort(labels, kind="stable")
    offsets = np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=C))])
    return perm, offsets


def permute_rows(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Rows in the permuted order: out[p] = x[perm[p]]."""
    return np.asarray(x)[perm]


def unpermute_rows(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse of :func:`permute_rows`: out[perm[p]] = y[p]."""
    out = np.empty_like(np.asarray(y))
    out[perm] = y
    return out
