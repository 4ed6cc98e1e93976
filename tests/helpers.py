"""Shared helpers for the parity tests: run the CUDA path on seeded inputs and
compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

from free_block_sparse_kv_b200 import workloads as W
from oracle import block_sparse_attention as O

# Output tolerance for floating point: max abs error and mean relative (L1 ratio) error.
MAX_ABS = 1e-2
MEAN_REL = 2e-3
# A kept-set decision is pinned (must match bit for bit) when the oracle's logit gap at
# the cutoff, and for mass routing both cumulative-mass margins, exceed this.
GATE = 1e-4

# Reduced workloads the oracle finishes in seconds. They keep each full workload's
# recipe and span several 64-wide tiles plus a ragged last block.
SMALL = {
    "uniform-4k": W.WORKLOADS["uniform-4k"],
    "dit-small": W.shrink(W.WORKLOADS["dit-21x30x52"], name="dit-small", H=2, Nq=9000, Nk=9000,
                          grid=(9, 20, 50)),
    "dit720p-small": W.shrink(W.WORKLOADS["dit720p-21x45x80"], name="dit720p-small", H=2, Nq=9480,
                              Nk=9480, grid=(6, 20, 79)),
    "longvideo-small": W.shrink(W.WORKLOADS["longvideo-41x30x52"], name="longvideo-small", H=2,
                                Nq=9500, Nk=9500, grid=(19, 10, 50), window=2, n_anchors=3,
                                period=6, steps=(0, 5)),
    "worldmodel-small": W.shrink(W.WORKLOADS["worldmodel-chunk"], name="worldmodel-small", B=2, H=2,
                                 Nq=500, Nk=6500, grid=(13, 10, 50), q_frame0=12),
    "longvideo-adaptive-small": W.shrink(W.WORKLOADS["longvideo-adaptive-41x30x52"],
                                         name="longvideo-adaptive-small", H=2, Nq=9500, Nk=9500,
                                         grid=(19, 10, 50), window=2, n_anchors=3, period=6,
                                         budget=9, steps=(0, 5)),
    "hybrid-small": W.shrink(W.WORKLOADS["dit720p-hybrid-21x45x80"], name="hybrid-small", H=2,
                             Nq=9480, Nk=9480, grid=(6, 20, 79)),
    "ear-small": W.shrink(W.WORKLOADS["dit720p-ear-21x45x80"], name="ear-small", H=2, Nq=9480,
                          Nk=9480, grid=(6, 20, 79)),
    "kmeans-small": W.shrink(W.WORKLOADS["dit720p-kmeans-21x45x80"], name="kmeans-small", H=2,
                             Nq=9480, Nk=9480, grid=(6, 20, 79), clusters=(38, 38, 3)),
    # error-aware routing on blocks cut from the k-means group-major order
    "ear-kmeans-small": W.shrink(W.WORKLOADS["dit720p-ear-21x45x80"], name="ear-kmeans-small", H=2,
                                 Nq=9480, Nk=9480, grid=(6, 20, 79), clusters=(38, 38, 3)),
}

# Error-aware scores (ln of the error per token). The GPU takes the logits with a 16-bit
# split of qbar and the weight differences with a 16-bit split (each within 2^-15 of
# its value) in fp32 arithmetic. The relative error of X (the block's numerator error,
# relative to the block's largest weight) is then a few 2^-16 / sqrt(3) per term, summed
# with random signs over the block, about 1e-5 of X where X >= EAR_X_FLOOR; the score is
# ln ||X||^2, so its error stays below EAR_TOL. A kept-set decision is pinned when the
# oracle's score gap at the cutoff exceeds two such errors.
EAR_X_FLOOR = 1e-2
EAR_TOL = 2e-4
EAR_GATE = 2 * EAR_TOL


def err_stats(got: np.ndarray, want: np.ndarray):
    diff = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    return float(diff.max()), float(diff.sum() / np.abs(want).sum())


def oracle_kept(w: W.Workload, q, k, step: int = 0, v=None):
    """Oracle kept lists of one head and the per-row gate flags (True = pinned).
    Covariance-aware and error-aware routing need the head's values ``v``."""
    if w.mode == "structured":
        kept = O.structured_kept(w.Nq, w.Nk, w.block, w.frame_tokens, w.n_frames, w.window,
                                 w.n_anchors, w.period, step, w.q_frame0, budget=w.budget)
        return kept, np.ones(len(kept), bool)
    if w.mode in ("topk", "topk_cov", "ear"):
        kept, s, counts = O.route_head(q, k, w.block, w.mode, w.scale, keep=w.keep(), v=v)
        gaps, _, _ = O.gate_diagnostics(s, counts)
        return kept, gaps > (EAR_GATE if w.mode == "ear" else GATE)
    kept, s, counts = O.route_head(q, k, w.block, "mass", w.scale, tau=w.tau)
    gaps, lo, hi = O.gate_diagnostics(s, counts, tau=w.tau)
    return kept, (gaps > GATE) & (lo > GATE) & (hi > GATE)


def oracle_layout(w: W.Workload, q, k, v):
    """The oracle's token layout of one head: (q', k', v', position of every original
    query row). Without clustering the layout is the given one."""
    if not w.clusters:
        return q, k, v, np.arange(q.shape[0])
    from oracle import cluster_layout as K
    cq, ck, iters = w.clusters
    lq, _ = K.kmeans(q, cq, iters)
    lk, _ = K.kmeans(k, ck, iters)
    pq, _ = K.group_major_permutation(lq, cq)
    pk, _ = K.group_major_permutation(lk, ck)
    pos = np.empty_like(pq)
    pos[pq] = np.arange(pq.shape[0])
    return K.permute_rows(q, pq), K.permute_rows(k, pk), K.permute_rows(v, pk), pos


def lists_to_sets(kv_idx: np.ndarray, kv_cnt: np.ndarray):
    return [sorted(int(x) for x in kv_idx[i, :kv_cnt[i]]) for i in range(kv_cnt.shape[0])]


def sample_rows(w: W.Workload, n: int, seed: int = 0):
    """Query rows to check at full size: first and last rows, both ends of the last
    (possibly partial) block, and a seeded spread in between."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, w.Nq - 1, w.Nq - 2, (w.nqb - 1) * w.block, min(w.Nq - 1, w.block)}
    rest = rng.choice(w.Nq, size=max(0, n - len(fixed)), replace=False)
    return np.array(sorted(fixed | set(int(x) for x in rest)))
