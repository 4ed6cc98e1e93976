"""Host-side logic of the benchmark (CPU only): the executed-flop model behind
`roofline.achieved`, the algorithmic pool bytes, the KV-cache offset of the world-model
chunk, the DRAM-traffic lookup and the peaks."""
import os

import numpy as np
import pytest

import bench
from free_block_sparse_kv_b200 import workloads as W


def _lists(w, kept):
    """kv_idx / kv_cnt arrays from one kept list per query block (same for every head)."""
    cap = max(1, max(len(k) for k in kept))
    idx = np.zeros((w.B, w.H, w.nqb, cap), np.int32)
    cnt = np.zeros((w.B, w.H, w.nqb), np.int32)
    for i, k in enumerate(kept):
        idx[:, :, i, :len(k)] = k
        cnt[:, :, i] = len(k)
    return idx, cnt


@pytest.mark.parametrize("order", [0, 1, 2])
def test_executed_flops_closed_forms(order):
    w = W.shrink(W.WORKLOADS["uniform-4k"], B=2, H=3, Nq=300, Nk=500, d=64, block=128,
                 order=order)
    nq = [128, 128, 44]
    nk = [128, 128, 128, 116]
    # everything kept: dense attention, 4 Nq Nk d per head
    f = bench.executed_flops(w, *_lists(w, [list(range(4))] * 3))
    assert f["exact"] == 6 * 4 * 300 * 500 * 64 and f["order0"] == f["order1"] == 0
    # nothing kept: every block compensated
    f = bench.executed_flops(w, *_lists(w, [[]] * 3))
    assert f["exact"] == 0
    assert f["order0"] == 6 * 4 * 300 * 64 * 4
    want1 = {0: 0, 1: 6 * 2 * 300 * 64 * 64 * 4, 2: 6 * 2 * 300 * 64 * 64}[order]
    assert f["order1"] == want1
    # mixed: query block i keeps block i (the last query and key blocks are partial)
    f = bench.executed_flops(w, *_lists(w, [[0], [1], [3]]))
    assert f["exact"] == 6 * 4 * 64 * sum(q * k for q, k in zip(nq, [nk[0], nk[1], nk[3]]))
    assert f["order0"] == 6 * 4 * 64 * 3 * 300
    assert f["total"] == f["exact"] + f["order0"] + f["order1"]


def test_pool_bytes_closed_form():
    w = W.shrink(W.WORKLOADS["uniform-4k"], B=1, H=2, Nq=256, Nk=512, d=64, block=128, order=1)
    bh, nkb, nqb = 2, 4, 2
    rd = bh * 512 * 64 * 2 * 2 + bh * 256 * 64 * 2
    # centroids and value sums: fp32 each plus one 16-bit copy each; query centroids fp32;
    # M_j in 16 bits
    wr = bh * nkb * 64 * 12 + bh * nqb * 64 * 4 + bh * nkb * 64 * 64 * 2
    assert bench.pool_bytes(w, True) == rd + wr
    assert bench.pool_bytes(w, False) == rd + wr - bh * 256 * 64 * 2 - bh * nqb * 64 * 4
    # what the library writes beyond the method's tables: the fp16 copy of V and the low
    # centroid plane
    assert bench.pool_extra_bytes(w) == {"v16": bh * 512 * 64 * 2, "kbar16_lo": bh * nkb * 64 * 2}


def test_pool_bytes_of_the_metric_workload():
    """The 720p call moves 3.145 GB through the pool by the method's tables (K, V, Q read;
    M_j 0.775 GB written); the fp16 copy of V adds 0.774 GB."""
    w = W.WORKLOADS[W.METRIC_WORKLOAD]
    assert abs(bench.pool_bytes(w, True) - 3.1448e9) < 1e6
    assert abs(bench.pool_extra_bytes(w)["v16"] - 0.7741e9) < 1e6


def test_reference_rows_per_step():
    assert bench.reference_rows_per_step(0.01, 12.0, 20) == 48
    assert bench.reference_rows_per_step(1.0, 12.0, 20) == 16
    assert bench.reference_rows_per_step(1e-4, 10.0, 5) % 16 == 0


def test_launch_counts():
    assert bench.launches_per_step(W.WORKLOADS["dit720p-21x45x80"], 1) == 3
    assert bench.launches_per_step(W.WORKLOADS["worldmodel-chunk"], 3) == 4
    assert bench.launches_per_step(W.WORKLOADS["dit720p-hybrid-21x45x80"], 1) == 5
    assert bench.launches_per_step(W.WORKLOADS["dit720p-ear-21x45x80"], 1) == 4
    assert bench.launches_per_step(W.WORKLOADS["dit720p-kmeans-21x45x80"], 1) == 3 + 2 * 31 + 4


def test_kv_cache_start_of_the_world_model_chunk():
    w = W.WORKLOADS["worldmodel-chunk"]
    assert bench.kv_cached_start(w) == 40 * 1560 // 64 == 975
    assert bench.kv_cached_start(W.WORKLOADS["dit720p-21x45x80"]) == 0


def test_traffic_only_from_a_capture_of_the_current_sources():
    """The DRAM bytes of the capture are reported while the forward's sources still hash to
    the capture's value, and None otherwise (or where there is no capture)."""
    w = W.WORKLOADS[W.METRIC_WORKLOAD]
    path = os.path.join(bench.ROOT, "profiles", f"forward_dram_{w.name}.md")
    t = bench.forward_traffic(w)
    if bench.forward_sources_sha256() in open(path).read():
        assert t is not None and 4.0e9 < t < 2.0e10
    else:
        assert t is None
    assert bench.forward_traffic(W.WORKLOADS["uniform-4k"]) is None   # no capture there


def test_peaks_are_positive():
    pk = bench.peaks()
    assert pk["source"] in ("measured", "fallback")
    assert pk["bf16"] > 0 and pk["bf16_sustained"] > 0 and pk["hbm"] > 0
