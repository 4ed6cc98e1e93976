"""Pins for the fp64 oracle: hand-derived values, closed forms, invariants, library
routines and brute force. Each check is chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
count for a partial block) fails at least one of them."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import block_sparse_attention as O
from free_block_sparse_kv_b200 import workloads as W


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# --- hand-derived worked examples --------------------------------------------

def test_golden_single_block(golden_dir):
    g = _load(golden_dir, "single_block_d2.json")
    q, k, v = (np.array(g[x], float) for x in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(g["d"])
    kbar, vsum, counts, mats = O.pool_keys_values(k, v, g["block"], 1)
    np.testing.assert_allclose(kbar, g["kbar"], atol=1e-15)
    np.testing.assert_allclose(vsum, g["vsum"], atol=1e-15)
    np.testing.assert_allclose(mats, g["M"], atol=1e-15)
    assert counts.tolist() == [2]
    skipped = [np.zeros(0, int)]
    o0 = O.forward_head(q, k, v, skipped, g["block"], 0, scale)
    o1 = O.forward_head(q, k, v, skipped, g["block"], 1, scale)
    ok = O.forward_head(q, k, v, [np.array([0])], g["block"], 1, scale)
    np.testing.assert_allclose(o0, g["out_order0_skipped"], atol=1e-14)
    np.testing.assert_allclose(o1, g["out_order1_skipped"], atol=1e-14)
    np.testing.assert_allclose(ok, g["out_kept"], atol=1e-14)


def test_golden_routing(golden_dir):
    g = _load(golden_dir, "routing_d4.json")
    q, k = np.array(g["q"], float), np.array(g["k"], float)
    scale = 1.0 / math.sqrt(g["d"])
    qbar = O.pool_queries(q, g["block"])
    kbar = O.pool_keys_values(k, np.zeros((k.shape[0], 1)), g["block"], 0)[0]
    s = O.routing_scores(qbar, kbar, scale)
    np.testing.assert_allclose(s, g["scores"], atol=1e-15)
    for kk, want in g["topk"].items():
        assert O.route_topk(s, int(kk))[0].tolist() == want
    for tau, want in g["mass"].items():
        kept, cnt = O.route_mass(s, float(tau))
        assert kept[0].tolist() == want and cnt[0] == len(want)
    gaps, _, _ = O.gate_diagnostics(s, [2])
    assert gaps[0] == pytest.approx(g["gap_top2"], abs=1e-15)
    gaps, _, _ = O.gate_diagnostics(s, [1])
    assert gaps[0] == 0.0


def test_golden_mass_margins(golden_dir):
    """Cumulative-mass margins at the cutoff of the mass rule, hand-derived (closed
    forms in the fixture), including k = 1 where the lower margin is undefined."""
    g = _load(golden_dir, "mass_margins_d4.json")
    s = np.array([g["scores"]], float)
    for case in g["cases"]:
        kept, cnt = O.route_mass(s, case["tau"])
        assert cnt[0] == case["k"]
        gaps, lo, hi = O.gate_diagnostics(s, cnt, tau=case["tau"])
        assert gaps[0] == pytest.approx(case["gap"], abs=1e-15)
        if case["lo"] == "inf":
            assert lo[0] == math.inf
        else:
            assert lo[0] == pytest.approx(case["lo"], abs=1e-12)
        assert hi[0] == pytest.approx(case["hi"], abs=1e-12)


def test_mass_margins_match_brute_force_sums():
    """Margins against an independent ranking (Python sort) and exactly rounded sums
    (math.fsum): tau - C_(k-1) > 0 >= tau - C_k, both reported with the right sign."""
    rng = np.random.default_rng(11)
    s = 1.5 * rng.standard_normal((30, 25))
    for tau in (0.3, 0.75, 0.95):
        _, counts = O.route_mass(s, tau)
        _, lo, hi = O.gate_diagnostics(s, counts, tau=tau)
        for i, row in enumerate(s):
            z = [math.exp(x - max(row)) for x in row]
            total = math.fsum(z)
            ranked = sorted(range(len(row)), key=lambda j: (-row[j], j))
            k = counts[i]
            c_k = math.fsum(z[j] for j in ranked[:k]) / total
            c_km1 = math.fsum(z[j] for j in ranked[:k - 1]) / total
            assert hi[i] == pytest.approx(c_k - tau, abs=1e-12) and hi[i] >= -1e-12
            if k == 1:
                assert lo[i] == math.inf
            else:
                assert lo[i] == pytest.approx(tau - c_km1, abs=1e-12) and lo[i] > 0


def test_golden_structured(golden_dir):
    g = _load(golden_dir, "structured_small.json")
    kept = O.structured_kept(g["Nq"], g["Nk"], g["block"], g["frame_tokens"], g["n_frames"],
                             g["window"], g["n_anchors"], g["period"], g["step"])
    assert [x.tolist() for x in kept] == g["kept"]


def test_golden_structured_adaptive(golden_dir):
    g = _load(golden_dir, "structured_adaptive.json")
    kept = O.structured_kept(g["Nq"], g["Nk"], g["block"], g["frame_tokens"], g["n_frames"],
                             g["window"], g["n_anchors"], g["period"], g["step"], budget=g["budget"])
    assert [x.tolist() for x in kept] == g["kept"]


@pytest.mark.parametrize("n_frames,window,n_anchors,period,budget", [
    (41, 3, 4, 10, 11), (41, 3, 4, 10, 21), (12, 0, 3, 4, 5), (9, 2, 2, 5, 40), (20, 1, 5, 4, 3)])
def test_adaptive_window_reaches_the_budget(n_frames, window, n_anchors, period, budget):
    for step in range(period):
        for t in range(n_frames):
            base = O.attend_frames(t, step, window, period, n_anchors, n_frames)
            ext = O.attend_frames(t, step, window, period, n_anchors, n_frames, budget)
            assert base <= ext
            assert len(ext) == max(len(base), min(budget, n_frames)), (step, t)
            assert t in ext


# --- rho = 1 is dense attention ----------------------------------------------

@pytest.mark.parametrize("order", [0, 1])
def test_all_kept_equals_dense_loops(order):
    rng = np.random.default_rng(1)
    n, d, b = 100, 8, 32                  # partial last block (4 tokens)
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    scale = 1 / math.sqrt(d)
    nb = -(-n // b)
    kept = [np.arange(nb)] * nb
    got = O.forward_head(q, k, v, kept, b, order, scale)
    want = O.dense_attention_loops(q, k, v, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_all_kept_equals_sdpa_at_small_workload_size():
    w = W.WORKLOADS["uniform-4k"]
    q, k, v = W.head_inputs(w, 0, 1)
    kept = [np.arange(w.nkb)] * w.nqb
    rows = np.arange(0, w.Nq, 37)
    got = O.forward_head(q, k, v, kept, w.block, 0, w.scale, rows=rows)
    qt, kt, vt = (torch.from_numpy(x.astype(np.float64)) for x in (q[rows], k, v))
    want = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None]).numpy()[0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# --- order-0 exactness and first-order convergence ----------------------------

def test_order0_exact_for_identical_keys_in_block():
    rng = np.random.default_rng(2)
    n, d, b = 200, 16, 32                 # 7 blocks, last holds 8 tokens
    nb = -(-n // b)
    centers = _rand(rng, nb, d)
    k = centers[np.arange(n) // b]
    q, v = _rand(rng, n, d), _rand(rng, n, d)
    scale = 1 / math.sqrt(d)
    _, _, counts, mats = O.pool_keys_values(k, v, b, 1)
    assert np.abs(mats).max() < 1e-12
    assert counts[-1] == n - (nb - 1) * b
    kept = [rng.choice(nb, size=2, replace=False) for _ in range(nb)]
    for order in (0, 1):
        got = O.forward_head(q, k, v, kept, b, order, scale)
        want = O.dense_attention_loops(q, k, v, scale)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_taylor_orders_converge_at_rate_one_and_two():
    rng = np.random.default_rng(3)
    n, d, b = 192, 16, 64
    nb = n // b
    centers = 0.5 * _rand(rng, nb, d)
    delta = _rand(rng, n, d)
    q, v = _rand(rng, n, d), _rand(rng, n, d)
    scale = 1 / math.sqrt(d)
    kept = [np.array([i]) for i in range(nb)]    # each query block keeps only itself
    errs = {0: [], 1: []}
    eps_list = [1e-1, 1e-2, 1e-3]
    for eps in eps_list:
        k = centers[np.arange(n) // b] + eps * delta
        dense = O.dense_attention_loops(q, k, v, scale)
        for order in (0, 1):
            errs[order].append(np.abs(O.forward_head(q, k, v, kept, b, order, scale) - dense).max())
    for order, want in ((0, 1.0), (1, 2.0)):
        slope = np.polyfit(np.log(eps_list), np.log(errs[order]), 1)[0]
        assert abs(slope - want) < 0.15, (order, slope, errs[order])
    assert errs[1][-1] < 1e-2 * errs[0][-1]


# --- pooled-table algebra vs the per-pair twin ---------------------------------

@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("rho", [(1, 4), (1, 2)])
def test_blockwise_equals_per_pair_twin(order, rho):
    rng = np.random.default_rng(10 + order)
    n, d, b = 300, 8, 32                  # 10 blocks, the last has 12 tokens
    q, k, v = _rand(rng, n, d), 0.5 * _rand(rng, n, d), _rand(rng, n, d)
    scale = 1 / math.sqrt(d)
    keep = O.keep_count(-(-n // b), *rho)
    kept, _, _ = O.route_head(q, k, b, "topk", scale, keep=keep)
    got = O.forward_head(q, k, v, kept, b, order, scale)
    want = O.brute_force_pairs(q, k, v, kept, b, order, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_all_skipped_order0_is_attention_over_pseudo_tokens():
    """With nothing kept, order 0 is attention over one pseudo-token per block: key
    kbar_j, value S_j / n_j and logit bias ln n_j (torch SDPA in fp64)."""
    rng = np.random.default_rng(4)
    n, d, b = 500, 32, 64                 # last block 52 tokens
    q, k, v = _rand(rng, n, d), _rand(rng, n, d), _rand(rng, n, d)
    scale = 1 / math.sqrt(d)
    nb = -(-n // b)
    got = O.forward_head(q, k, v, [np.zeros(0, int)] * nb, b, 0, scale)
    kb = np.stack([k[s:s + b].mean(0) for s in range(0, n, b)])
    vm = np.stack([v[s:s + b].mean(0) for s in range(0, n, b)])
    cnt = np.array([min(b, n - s) for s in range(0, n, b)], float)
    bias = torch.from_numpy(np.log(cnt))[None, :].expand(n, nb)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(kb)[None], torch.from_numpy(vm)[None],
        attn_mask=bias[None]).numpy()[0]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# --- routing -----------------------------------------------------------------

def test_topk_matches_rank_counting():
    rng = np.random.default_rng(5)
    s = np.round(rng.standard_normal((40, 37)), 1)     # many exact ties
    keep = 9
    kept = O.route_topk(s, keep)
    for i, row in enumerate(s):
        rank = [sum(1 for jj in range(len(row)) if row[jj] > row[j] or (row[jj] == row[j] and jj < j))
                for j in range(len(row))]
        assert kept[i].tolist() == [j for j in range(len(row)) if rank[j] < keep]


def test_mass_prefix_is_shortest_covering():
    rng = np.random.default_rng(6)
    s = 2.0 * rng.standard_normal((50, 60))
    for tau in (0.5, 0.9, 0.99):
        kept, counts = O.route_mass(s, tau)
        for i, row in enumerate(s):
            z = [math.exp(x) for x in row]
            total = math.fsum(z)
            ranked = sorted(range(len(row)), key=lambda j: (-row[j], j))
            k = counts[i]
            assert math.fsum(z[j] for j in ranked[:k]) / total >= tau - 1e-12
            assert math.fsum(z[j] for j in ranked[:k - 1]) / total < tau
            assert kept[i].tolist() == sorted(ranked[:k])


def test_keep_count_is_integer_ceiling():
    assert O.keep_count(64, 1, 4) == 16
    assert O.keep_count(256, 1, 5) == 52
    assert O.keep_count(591, 1, 10) == 60
    assert O.keep_count(10, 1, 1) == 10


# --- structured mask ---------------------------------------------------------

def test_rotating_anchors_cover_each_frame_once():
    period, n_anchors, n_frames = 10, 4, 41
    seen = {}
    for s in range(period):
        for f in O.anchor_frames(s, period, n_anchors, n_frames):
            seen[f] = seen.get(f, 0) + 1
    assert sorted(seen) == list(range(40)) and set(seen.values()) == {1}
    assert O.anchor_frames(3, period, n_anchors, n_frames) == O.anchor_frames(13, period, n_anchors, n_frames)


def test_structured_mask_against_token_pairs():
    """Brute force over every (query token, key token) pair on a geometry whose
    blocks straddle frame boundaries."""
    ft, T, b, win, na, per = 7, 9, 5, 1, 2, 4
    n = ft * T
    for step in range(per):
        kept = O.structured_kept(n, n, b, ft, T, win, na, per, step)
        anchors = {(step % per) + per * m for m in range(na)}
        for i in range(-(-n // b)):
            want = []
            for j in range(-(-n // b)):
                hit = False
                for tq in range(i * b, min(n, (i + 1) * b)):
                    for tk in range(j * b, min(n, (j + 1) * b)):
                        fq, fk = tq // ft, tk // ft
                        if abs(fq - fk) <= win or fk in anchors:
                            hit = True
                want.append(hit)
            assert kept[i].tolist() == [j for j, h in enumerate(want) if h]


def test_structured_mask_of_a_query_chunk_against_token_pairs():
    """A query chunk that starts mid-video (q_frame0 > 0, an autoregressive chunk):
    query token t lies in frame q_frame0 + t // frame_tokens. Brute force over every
    (query token, key token) pair, with blocks that straddle frames on both sides."""
    ft, T, b, win, na, per = 7, 9, 5, 1, 2, 4
    nk = ft * T
    for q_frame0, nq in ((4, 17), (6, 21), (8, 7)):
        for step in (0, 3):
            kept = O.structured_kept(nq, nk, b, ft, T, win, na, per, step, q_frame0=q_frame0)
            anchors = {(step % per) + per * m for m in range(na)}
            assert len(kept) == -(-nq // b)
            for i in range(-(-nq // b)):
                want = []
                for j in range(-(-nk // b)):
                    hit = False
                    for tq in range(i * b, min(nq, (i + 1) * b)):
                        for tk in range(j * b, min(nk, (j + 1) * b)):
                            fq, fk = q_frame0 + tq // ft, tk // ft
                            if abs(fq - fk) <= win or fk in anchors:
                                hit = True
                    want.append(hit)
                assert kept[i].tolist() == [j for j, h in enumerate(want) if h]


@pytest.mark.parametrize("budget", [0, 6])
def test_structured_mask_of_a_chunk_equals_the_rows_of_the_whole_video(budget):
    """When a chunk starts on a block boundary, its query blocks are blocks of the whole
    video: the chunk's mask (q_frame0 > 0) equals those rows of the full mask, with and
    without adaptive windows."""
    ft, T, b, win, na, per = 6, 10, 3, 1, 2, 5
    full = O.structured_kept(ft * T, ft * T, b, ft, T, win, na, per, 2, budget=budget)
    for f0, nframes in ((2, 2), (5, 3), (9, 1)):
        chunk = O.structured_kept(ft * nframes, ft * T, b, ft, T, win, na, per, 2, q_frame0=f0,
                                  budget=budget)
        first = f0 * ft // b
        assert [x.tolist() for x in chunk] == [x.tolist() for x in full[first:first + len(chunk)]]


def test_structured_kept_fraction_at_long_video_size():
    """At 41 frames x 1560 tokens, blocks of 128, window 3, 4 anchors: a query frame
    sees its clipped window plus the anchors outside it; block granularity adds
    the straddling blocks. The kept fraction lies between the frame-level pair
    fraction and that fraction plus two boundary blocks per row."""
    w = W.WORKLOADS["longvideo-41x30x52"]
    T = w.n_frames
    for step in (0, 7):
        kept = O.structured_kept(w.Nq, w.Nk, w.block, w.frame_tokens, T, w.window,
                                 w.n_anchors, w.period, step)
        frac = sum(len(x) for x in kept) / (w.nqb * w.nkb)
        g = {(step % w.period) + w.period * m for m in range(w.n_anchors)}
        pairs = sum(len(g | {f for f in range(t - 3, t + 4) if 0 <= f < T}) for t in range(T))
        lo = pairs / T ** 2
        assert lo <= frac <= lo + 2 * (1 + len(g)) * 2 / w.nkb + 2 / w.nkb


def test_mass_boundary_is_inclusive(golden_dir):
    g = _load(golden_dir, "routing_d4.json")
    kept, cnt = O.route_mass(np.array(g["equal_scores"]), g["equal_scores_tau"])
    assert kept[0].tolist() == g["equal_scores_kept"] and cnt[0] == 2


# ---------------------------------------------------------------------------
# Hybrid order (global first-order matrix) and covariance-aware routing
# ---------------------------------------------------------------------------

def _shared_deviation_head(n_blocks, block, d, seed, sign=None):
    """Keys c_j + e_r and values s_j * w_r: every block has the same deviations e_r
    (summing to zero over the block) and the same values up to a sign s_j, so
    M_j = s_j * sum_r e_r w_r^T is one matrix for all blocks (or its negative)."""
    rng = np.random.default_rng(seed)
    e = rng.standard_normal((block, d))
    e -= e.mean(axis=0)
    w = rng.standard_normal((block, d))
    sign = np.ones(n_blocks) if sign is None else np.asarray(sign, float)
    centers = rng.standard_normal((n_blocks, d))
    k = np.concatenate([centers[j] + e for j in range(n_blocks)])
    v = np.concatenate([sign[j] * w for j in range(n_blocks)])
    q = rng.standard_normal((n_blocks * block, d))
    return q, k, v


def test_hybrid_equals_per_block_order1_when_blocks_share_their_first_order_matrix():
    q, k, v = _shared_deviation_head(4, 16, 8, seed=11)
    kbar, vsum, counts, mats = O.pool_keys_values(k, v, 16, 1)
    np.testing.assert_allclose(mats, np.broadcast_to(mats[0], mats.shape), atol=1e-12)
    np.testing.assert_allclose(O.global_first_order(mats), mats[0], atol=1e-12)
    kept = [np.array([i]) for i in range(4)]
    o1 = O.forward_head(q, k, v, kept, 16, 1, 0.3)
    o2 = O.forward_head(q, k, v, kept, 16, 2, 0.3)
    o0 = O.forward_head(q, k, v, kept, 16, 0, 0.3)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    assert np.abs(o2 - o0).max() > 1e-3  # the first-order term is present


def test_hybrid_equals_order0_when_the_mean_first_order_matrix_vanishes():
    q, k, v = _shared_deviation_head(4, 16, 8, seed=12, sign=[1, -1, 1, -1])
    _, _, _, mats = O.pool_keys_values(k, v, 16, 1)
    np.testing.assert_allclose(O.global_first_order(mats), 0.0, atol=1e-12)
    kept = [np.array([i]) for i in range(4)]
    np.testing.assert_allclose(O.forward_head(q, k, v, kept, 16, 2, 0.3),
                               O.forward_head(q, k, v, kept, 16, 0, 0.3), atol=1e-12)


def test_covariance_norms_hand_example():
    # block 1: keys (+-1, 0), values (+-1/2, 0) -> M_1 = [[1, 0], [0, 0]]
    # block 2: keys (0, +-1), values (0, +-1/2) -> M_2 = [[0, 0], [0, 1]]
    k = np.array([[1.0, 0.0], [-1.0, 0.0], [0.0, 1.0], [0.0, -1.0]])
    v = np.array([[0.5, 0.0], [-0.5, 0.0], [0.0, 0.5], [0.0, -0.5]])
    _, _, _, mats = O.pool_keys_values(k, v, 2, 1)
    np.testing.assert_allclose(mats[0], [[1, 0], [0, 0]], atol=1e-15)
    np.testing.assert_allclose(mats[1], [[0, 0], [0, 1]], atol=1e-15)
    hbar = O.global_first_order(mats)
    np.testing.assert_allclose(hbar, [[0.5, 0], [0, 0.5]], atol=1e-15)
    np.testing.assert_allclose(O.covariance_norms(mats, hbar), [math.sqrt(0.5)] * 2, atol=1e-15)


def test_covariance_score_can_overtake_the_attention_score():
    # scores 1.0 and 0.9; norms 1 and e: the second block gains ln e = 1 and wins top-1
    s = np.array([[1.0, 0.9]])
    c = np.array([1.0, math.e])
    cs = O.covariance_scores(s, c)
    np.testing.assert_allclose(cs, [[1.0, 1.9]], atol=1e-15)
    assert [list(x) for x in O.route_topk(cs, 1)] == [[1]]
    assert [list(x) for x in O.route_topk(s, 1)] == [[0]]


# --- error-aware routing (SVG-EAR §2 B) -----------------------------------------

def test_golden_ear(golden_dir):
    g = _load(golden_dir, "ear_d2.json")
    q, k, v = (np.array(g[x], float) for x in ("q", "k", "v"))
    qbar = O.pool_queries(q, g["block"])
    got = O.ear_scores(qbar, k, v, g["block"], g["scale"])
    want = np.array([[float(x) for x in row] for row in g["scores"]])
    assert got.shape == want.shape
    np.testing.assert_allclose(got[:, 0], want[:, 0], rtol=0, atol=1e-12)
    assert np.isneginf(got[0, 1])


def test_ear_constant_values_reduce_to_the_denominator_gap():
    # With v_r = u for every token of the block, the numerator error is u times the
    # scalar gap sum_r exp(s_r) - n exp(s_c), which is >= 0 by Jensen's inequality.
    rng = np.random.default_rng(11)
    block, d, scale = 8, 4, 0.5
    k = _rand(rng, 24, d)
    u = _rand(rng, d)
    v = np.tile(u, (24, 1))
    qbar = _rand(rng, 3, d)
    got = O.ear_scores(qbar, k, v, block, scale)
    for j in range(3):
        kb = k[block * j:block * (j + 1)]
        for i in range(3):
            gap = np.exp(scale * kb @ qbar[i]).sum() - block * np.exp(scale * kb.mean(0) @ qbar[i])
            assert gap > 0
            want = 2 * np.log(gap) + np.log(u @ u) - np.log(block)
            assert abs(got[i, j] - want) < 1e-10


def test_ear_invariants():
    rng = np.random.default_rng(12)
    block, d, scale = 16, 8, 0.35
    k, v = _rand(rng, 40, d), _rand(rng, 40, d)
    qbar = _rand(rng, 5, d)
    base = O.ear_scores(qbar, k, v, block, scale)
    assert np.all(np.isfinite(base))
    # values scaled by c: error scaled by c^2
    np.testing.assert_allclose(O.ear_scores(qbar, k, 3.0 * v, block, scale), base + 2 * np.log(3.0),
                               atol=1e-10)
    # one key shift delta for every token of block 1: every logit of the block, the
    # centroid's included, moves by scale * qbar.delta, so the error moves by twice that
    delta = _rand(rng, d)
    k2 = k.copy()
    k2[16:32] += delta
    got = O.ear_scores(qbar, k2, v, block, scale)
    np.testing.assert_allclose(got[:, 1], base[:, 1] + 2 * scale * qbar @ delta, atol=1e-9)
    np.testing.assert_allclose(got[:, [0, 2]], base[:, [0, 2]], atol=1e-12)
    # the tokens' order inside a block does not matter
    perm = np.concatenate([rng.permutation(16), 16 + rng.permutation(16), 32 + rng.permutation(8)])
    np.testing.assert_allclose(O.ear_scores(qbar, k[perm], v[perm], block, scale), base, atol=1e-10)


def test_ear_error_vanishes_for_keys_the_proxy_cannot_tell_apart():
    # keys that differ only orthogonally to qbar give every token the centroid's logit
    rng = np.random.default_rng(13)
    d, block = 4, 8
    qbar = np.array([[1.0, 0.0, 0.0, 0.0]])
    k = _rand(rng, 16, d)
    k[:8, 0] = 0.7
    v = _rand(rng, 16, d)
    got = O.ear_scores(qbar, k, v, block, 1.0)
    assert got[0, 0] < got[0, 1] - 20 or np.isneginf(got[0, 0])
    k[:8] = k[0]
    assert np.isneginf(O.ear_scores(qbar, k, v, block, 1.0)[0, 0])


def test_ear_prefers_a_heterogeneous_block_over_a_high_score_homogeneous_one():
    # SVG-EAR §2 B: a block with a high attention score can be well approximated by its
    # centroid, a low-score block with heterogeneous keys cannot.
    rng = np.random.default_rng(14)
    d, block = 8, 16
    qbar = np.zeros((1, d))
    qbar[0, 0] = 2.0
    k = np.zeros((32, d))
    k[:16] = 1.0 + 0.01 * _rand(rng, 16, d)     # high score, nearly identical keys
    k[16:] = 0.3 * _rand(rng, 16, d)            # low score, spread-out keys
    k[16:, 0] += 0.2
    v = _rand(rng, 32, d)
    scale = 0.5
    att = O.routing_scores(qbar, np.stack([k[:16].mean(0), k[16:].mean(0)]), scale)
    ear = O.ear_scores(qbar, k, v, block, scale)
    assert att[0, 0] > att[0, 1]
    assert ear[0, 1] > ear[0, 0]
    kept_att = O.route_head(np.tile(qbar, (block, 1)), k, block, "topk", scale, keep=1)[0][0]
    kept_ear = O.route_head(np.tile(qbar, (block, 1)), k, block, "ear", scale, keep=1, v=v)[0][0]
    assert kept_att.tolist() == [0] and kept_ear.tolist() == [1]


def test_ear_divides_the_error_by_the_block_size():
    # Block 0 holds every token of the partial block 1 twice: the numerator error doubles
    # in amplitude (x4 squared) while the cost doubles, so the scores differ by ln 2.
    rng = np.random.default_rng(15)
    d = 4
    kb, vb = _rand(rng, 4, d), _rand(rng, 4, d)
    k = np.concatenate([np.repeat(kb, 2, axis=0), kb])   # block 0: 8 tokens, block 1: 4
    v = np.concatenate([np.repeat(vb, 2, axis=0), vb])
    qbar = _rand(rng, 2, d)
    got = O.ear_scores(qbar, k, v, 8, 0.5)
    np.testing.assert_allclose(got[:, 0] - got[:, 1], np.log(4.0) - np.log(2.0), atol=1e-10)
