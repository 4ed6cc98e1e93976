"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded inputs.

Masks: bit-exact wherever the oracle's cutoff gap exceeds the gate. Outputs: max
abs error and mean relative error within the stated tolerance, on fp32 output.
"""
import numpy as np
import pytest
import torch

from free_block_sparse_kv_b200 import attention as A
from free_block_sparse_kv_b200 import sparse_attn as C
from free_block_sparse_kv_b200 import workloads as W
from oracle import block_sparse_attention as O
from tests.helpers import (EAR_TOL, EAR_X_FLOOR, GATE, MAX_ABS, MEAN_REL, SMALL, err_stats,
                           lists_to_sets, oracle_kept, oracle_layout, sample_rows)

pytestmark = pytest.mark.gpu


def _dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _problem(w):
    return A.Problem(w.B, w.H, w.Nq, w.Nk, w.d, w.block, w.order)


def _geometry(w):
    return dict(frame_tokens=w.frame_tokens, n_frames=w.n_frames, window=w.window,
                n_anchors=w.n_anchors, period=w.period, q_frame0=w.q_frame0, budget=w.budget)


def _run(w, q, k, v, step=0, out_dtype=torch.float32):
    op = A.BlockSparseAttention(_problem(w), w.mode, rho=w.rho, tau=w.tau,
                                geometry=_geometry(w) if w.mode == "structured" else None,
                                out_dtype=out_dtype, clusters=w.clusters or None)
    out = op(q, k, v, step=step)
    torch.cuda.synchronize()
    op.check()
    return op, out


def _sample_rows_small(w, per_tile=3, seed=1):
    rng = np.random.default_rng(seed)
    rows = set()
    for s in range(0, w.Nq, 64):
        e = min(w.Nq, s + 64)
        rows |= {s, e - 1}
        rows |= set(int(x) for x in rng.integers(s, e, size=per_tile))
    return np.array(sorted(rows))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


@pytest.fixture(scope="module")
def small_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            w = SMALL[name]
            cache[name] = (w,) + W.full_inputs_bits(w)
        return cache[name]
    return get


# --- pooling -------------------------------------------------------------------

@pytest.mark.parametrize("name", list(SMALL))
def test_pool_matches_oracle(name, small_inputs):
    w, qb, kb, vb = small_inputs(name)
    p = _problem(w)
    t = A.allocate_tables(p, "cuda")
    A.pool(_dev(qb), _dev(kb), _dev(vb), p, t)
    torch.cuda.synchronize()
    for b in range(w.B):
        for h in range(w.H):
            q, k, v = (W.bits_to_f32(x[b, h]) for x in (qb, kb, vb))
            kbar, vsum, counts, mats = O.pool_keys_values(k, v, w.block, w.order)
            qbar = O.pool_queries(q, w.block)
            np.testing.assert_allclose(t.qbar[b, h].cpu().numpy(), qbar, rtol=0, atol=2e-6)
            np.testing.assert_allclose(t.kbar_t[b, h].cpu().numpy().T, kbar, rtol=0, atol=2e-6)
            np.testing.assert_allclose(t.vsum[b, h].cpu().numpy(), vsum, rtol=0, atol=2e-5)
            hi = t.kbar16[b, h, 0].double().cpu().numpy()
            lo = t.kbar16[b, h, 1].double().cpu().numpy()
            np.testing.assert_allclose(hi, kbar, rtol=2 ** -8, atol=1e-30)
            np.testing.assert_allclose(hi + lo, kbar, rtol=2 ** -15, atol=1e-7)
            v16 = t.vsum16[b, h].float().cpu().numpy()
            np.testing.assert_allclose(v16, vsum, rtol=2 ** -10, atol=1e-5)
            v16 = t.v16[b, h].float().cpu().numpy()
            # fp16 rounding of V (round to nearest even; exact except for subnormals)
            assert np.array_equal(v16, v.astype(np.float16).astype(np.float32))
            if w.order >= 1:
                mg = t.M[b, h].float().cpu().numpy()
                tol = 2 ** -10 * np.abs(mats) + 1e-3
                assert np.all(np.abs(mg - mats) <= tol), float(np.abs(mg - mats).max())
            if w.order == 2:
                # mean of the fp16 M table: each entry within the table's rounding
                hbar = O.global_first_order(mats)
                err = np.abs(t.hbar[b, h].cpu().numpy() - hbar)
                assert err.max() <= 2 ** -11 * np.abs(mats).max() + 1e-5, float(err.max())
                np.testing.assert_array_equal(t.hbar16[b, h].cpu().numpy(),
                                              t.hbar[b, h].cpu().numpy().astype(np.float16))
                cov = O.covariance_norms(mats, hbar)
                np.testing.assert_allclose(t.cov[b, h].cpu().numpy(), cov, rtol=1e-3)


# --- routing and structured masks ----------------------------------------------

@pytest.mark.parametrize("name", [n for n, w in SMALL.items() if w.mode != "structured"])
def test_route_masks_bit_exact_above_gate(name, small_inputs):
    w, qb, kb, vb = small_inputs(name)
    op, _ = _run(w, _dev(qb), _dev(kb), _dev(vb))
    idx, cnt = op.kv_idx.cpu().numpy(), op.kv_cnt.cpu().numpy()
    pinned = total = 0
    for b in range(w.B):
        for h in range(w.H):
            q, k, v, _ = oracle_layout(w, *(W.bits_to_f32(x[b, h]) for x in (qb, kb, vb)))
            kept, gate = oracle_kept(w, q, k, v=v)
            got = lists_to_sets(idx[b, h], cnt[b, h])
            for i in range(w.nqb):
                total += 1
                if w.mode in ("topk", "topk_cov", "ear"):
                    assert len(got[i]) == w.keep()
                if gate[i]:
                    pinned += 1
                    assert got[i] == kept[i].tolist(), (b, h, i)
    assert pinned >= 0.5 * total, (pinned, total)


@pytest.mark.parametrize("name", ["longvideo-small", "longvideo-41x30x52", "worldmodel-chunk",
                                  "longvideo-adaptive-small", "longvideo-adaptive-41x30x52"])
@pytest.mark.parametrize("budget", [None, 0, 6, 40])
def test_structured_mask_bit_exact(name, budget):
    w = SMALL.get(name) or W.WORKLOADS[name]
    budget = w.budget if budget is None else budget
    p = A.Problem(1, 2, w.Nq, w.Nk, w.d, w.block, w.order)
    steps = range(w.period) if w.mode == "structured" else (0, 3)
    for step in steps:
        idx, cnt = A.allocate_lists(p, p.nkb, "cuda")
        A.structured_mask(p, idx, cnt, w.frame_tokens, w.n_frames, w.window, w.n_anchors,
                          w.period, step, w.q_frame0, budget=budget)
        torch.cuda.synchronize()
        want = O.structured_kept(w.Nq, w.Nk, w.block, w.frame_tokens, w.n_frames, w.window,
                                 w.n_anchors, w.period, step, w.q_frame0, budget=budget)
        for h in range(2):
            got = lists_to_sets(idx[0, h].cpu().numpy(), cnt[0, h].cpu().numpy())
            assert got == [x.tolist() for x in want], (name, step)


# --- error-aware routing scores ---------------------------------------------------

def _ear_check(scores_gpu, q, k, v, block, scale):
    """GPU scores of one head against the oracle: within EAR_TOL wherever the block's
    relative error X is above the floor, and small (or -inf) on both sides below it."""
    qbar = O.pool_queries(q, block)
    want = O.ear_scores(qbar, k, v, block, scale)
    got = np.asarray(scores_gpu, np.float64)
    assert not np.isnan(got).any()
    # X relative to the block's largest weight: err = X^2 exp(2 m), score = ln(err / n)
    m = np.stack([(scale * (qbar @ k[s:e].T)).max(axis=1)
                  for s, e in O.block_ranges(k.shape[0], block)], axis=1)
    n = np.array([e - s for s, e in O.block_ranges(k.shape[0], block)], np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        x_want = np.exp(0.5 * (want + np.log(n)) - m)
        x_got = np.exp(0.5 * (got + np.log(n)) - m)
    big = x_want >= EAR_X_FLOOR
    assert big.mean() > 0.5, big.mean()
    err = np.abs(got[big] - want[big])
    assert err.max() <= EAR_TOL, float(err.max())
    assert np.all(x_got[~big] <= 2 * EAR_X_FLOOR), float(x_got[~big].max())
    return err.max()


@pytest.mark.parametrize("d,block,Nq,Nk", [(64, 64, 700, 4097), (64, 128, 3000, 6500),
                                           (128, 64, 300, 6401), (128, 128, 9000, 1000),
                                           (128, 128, 128, 100)])
def test_ear_scores_match_oracle(d, block, Nq, Nk):
    """Random inputs: several centroid tiles (the last partial), several runs of key
    blocks (the last partial), a ragged last key block (one token where Nk % block == 1,
    whose score is -inf on both sides) and a single partial block."""
    B, H = 1, 2
    qb, kb, vb = (_rand_bits((B, H, N, d), s) for N, s in ((Nq, 21), (Nk, 22), (Nk, 23)))
    p = A.Problem(B, H, Nq, Nk, d, block, 0)
    t = A.allocate_tables(p, "cuda", ear=True)
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.pool(q_d, k_d, v_d, p, t)
    A.ear_scores(k_d, v_d, p, t, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        got = t.scores[0, h].cpu().numpy()
        _ear_check(got, q, k, v, block, 1 / np.sqrt(d))
        if Nk % block == 1:
            assert np.all(np.isneginf(got[:, -1]))


def test_ear_scores_match_oracle_on_the_workload(small_inputs):
    w, qb, kb, vb = small_inputs("ear-small")
    op, _ = _run(w, _dev(qb), _dev(kb), _dev(vb))
    for b in range(w.B):
        for h in range(w.H):
            q, k, v = (W.bits_to_f32(x[b, h]) for x in (qb, kb, vb))
            _ear_check(op.tables.scores[b, h].cpu().numpy(), q, k, v, w.block, w.scale)


def test_route_scores_selects_like_the_oracle_on_given_scores():
    """Top-k over given scores is integer work: exact against the oracle's selection,
    with many exact ties, -inf entries and a keep count that splits tied groups."""
    B, H, nqb, nkb = 1, 3, 37, 300
    rng = np.random.default_rng(31)
    s = rng.integers(0, 40, size=(B, H, nqb, nkb)).astype(np.float32) * np.float32(0.25)
    s[rng.random(s.shape) < 0.1] = -np.inf
    s[0, 2] = -np.inf                            # a head where every score is -inf
    scores = torch.from_numpy(s).cuda()
    for rho in ((1, 10), (1, 3), (1, 1)):
        keep = -(-rho[0] * nkb // rho[1])
        idx = torch.zeros(B, H, nqb, keep, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, H, nqb, dtype=torch.int32, device="cuda")
        C.sparse_attn_route_scores(scores, B, H, nqb, nkb, rho[0], rho[1], idx, cnt, keep)
        torch.cuda.synchronize()
        for h in range(H):
            want = O.route_topk(s[0, h].astype(np.float64), keep)
            got = lists_to_sets(idx[0, h].cpu().numpy(), cnt[0, h].cpu().numpy())
            assert got == [x.tolist() for x in want], (rho, h)


# --- k-means and the group-major layout ---------------------------------------------

def _kmeans_check(xb, C, iters, B, H):
    """GPU k-means of bf16 rows xb [B,H,N,d] against the oracle, bit for bit."""
    from oracle import cluster_layout as K
    N, d = xb.shape[2], xb.shape[3]
    cl = A.allocate_clustering(B, H, N, d, C, iters, "cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = _dev(xb)
    A.kmeans(x, cl, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for b in range(B):
        for h in range(H):
            xf = W.bits_to_f32(xb[b, h])
            lab, cen = K.kmeans(xf, C, iters)
            perm, offs = K.group_major_permutation(lab, C)
            assert np.array_equal(cl.labels[b, h].cpu().numpy(), lab), (b, h)
            assert np.array_equal(cl.perm[b, h].cpu().numpy(), perm), (b, h)
            assert np.array_equal(cl.offsets[b, h].cpu().numpy(), offs), (b, h)
            assert np.array_equal(cl.centroids[b, h].cpu().numpy(), cen), (b, h)
    return cl, x


@pytest.mark.parametrize("d,N,C,iters", [(64, 700, 5, 0), (64, 3000, 130, 2), (128, 4097, 300, 3),
                                         (128, 1000, 1, 2), (128, 129, 129, 1)])
def test_kmeans_matches_oracle(d, N, C, iters):
    """Several token tiles (the last partial), several centroid tiles (the last partial),
    one cluster, as many clusters as tokens."""
    _kmeans_check(_rand_bits((1, 2, N, d), 40 + d + N), C, iters, 1, 2)


def test_kmeans_ties_and_empty_clusters():
    """Duplicated tokens: the initial centroids coincide, ties go to the lower index and
    the higher one is left empty and keeps its position."""
    rng = np.random.default_rng(41)
    base = rng.standard_normal((25, 64)).astype(np.float32)
    xb = W.bf16_round(np.repeat(base, 8, axis=0))[1][None, None]
    cl, _ = _kmeans_check(xb, 50, 2, 1, 1)
    offs = cl.offsets[0, 0].cpu().numpy()
    assert (np.diff(offs) == 0).any()


def test_kmeans_on_the_workload(small_inputs):
    w, qb, kb, _ = small_inputs("kmeans-small")
    cq, ck, iters = w.clusters
    _kmeans_check(qb, cq, iters, w.B, w.H)
    _kmeans_check(kb, ck, iters, w.B, w.H)


def test_permute_rows_round_trip():
    B, H, N, d = 1, 3, 777, 128
    xb = _rand_bits((B, H, N, d), 42)
    x = _dev(xb)
    rng = np.random.default_rng(43)
    perm = torch.from_numpy(np.stack([rng.permutation(N) for _ in range(B * H)]).reshape(B, H, N)
                            .astype(np.int32)).cuda()
    y = torch.empty_like(x)
    z = torch.empty_like(x)
    A.permute_rows(x, perm, y, gather=True)
    A.permute_rows(y, perm, z, gather=False)
    f = torch.randn(B, H, N, d, device="cuda")
    g, f2 = torch.empty_like(f), torch.empty_like(f)
    A.permute_rows(f, perm, g, gather=True)
    A.permute_rows(g, perm, f2, gather=False)
    torch.cuda.synchronize()
    pn = perm.cpu().numpy()
    assert torch.equal(z, x) and torch.equal(f2, f)
    assert np.array_equal(y.view(torch.int16).cpu().numpy()[0, 1], xb.view(np.int16)[0, 1][pn[0, 1]])


# --- forward ------------------------------------------------------------------

def _oracle_lists_to_device(w, kept_per_head, cap):
    idx = np.zeros((w.B, w.H, w.nqb, max(cap, 1)), np.int32)
    cnt = np.zeros((w.B, w.H, w.nqb), np.int32)
    for (b, h), kept in kept_per_head.items():
        for i, row in enumerate(kept):
            idx[b, h, i, :len(row)] = row
            cnt[b, h, i] = len(row)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle_on_oracle_masks(name, out_dtype, small_inputs):
    """Forward alone: the GPU forward consumes the oracle's kept lists."""
    w, qb, kb, vb = small_inputs(name)
    step = w.steps[-1] if w.mode == "structured" else 0
    kept_all = {}
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    for b, h in heads:
        q, k, v = (W.bits_to_f32(x[b, h]) for x in (qb, kb, vb))
        kept_all[(b, h)] = oracle_kept(w, q, k, step, v=v)[0]
    cap = max(len(r) for kept in kept_all.values() for r in kept)
    idx, cnt = _oracle_lists_to_device(w, kept_all, cap)
    p = _problem(w)
    t = A.allocate_tables(p, "cuda")
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    A.pool(q_d, k_d, v_d, p, t)
    out = torch.empty(w.B, w.H, w.Nq, w.d, dtype=out_dtype, device="cuda")
    A.forward(q_d, k_d, v_d, p, t, idx, cnt, out)
    torch.cuda.synchronize()
    rows = _sample_rows_small(w)
    got_all, want_all = [], []
    for b, h in heads:
        q, k, v = (W.bits_to_f32(x[b, h]) for x in (qb, kb, vb))
        want_all.append(O.forward_head(q, k, v, kept_all[(b, h)], w.block, w.order, w.scale,
                                       rows=rows))
        got_all.append(out[b, h, rows].float().cpu().numpy())
    got, want = np.concatenate(got_all), np.concatenate(want_all)
    mx, mr = err_stats(got, want)
    if out_dtype == torch.float32:
        assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)
    else:
        want16 = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
        floor = err_stats(want16, want)[1]
        assert mx <= MAX_ABS and mr <= MEAN_REL + floor, (mx, mr, floor)


@pytest.mark.parametrize("name", list(SMALL))
def test_pipeline_matches_oracle(name, small_inputs):
    """pool -> route (or mask) -> forward on the GPU against the oracle's own pipeline."""
    w, qb, kb, vb = small_inputs(name)
    steps = w.steps if w.mode == "structured" else (0,)
    rows = _sample_rows_small(w, per_tile=2, seed=2)
    for step in steps:
        _, out = _run(w, _dev(qb), _dev(kb), _dev(vb), step=step)
        got_all, want_all = [], []
        for b in range(w.B):
            for h in range(w.H):
                q, k, v, pos = oracle_layout(w, *(W.bits_to_f32(x[b, h]) for x in (qb, kb, vb)))
                kept, _ = oracle_kept(w, q, k, step, v=v)
                want_all.append(O.forward_head(q, k, v, kept, w.block, w.order, w.scale,
                                               rows=pos[rows]))
                got_all.append(out[b, h, rows].cpu().numpy())
        mx, mr = err_stats(np.concatenate(got_all), np.concatenate(want_all))
        assert mx <= MAX_ABS and mr <= MEAN_REL, (name, step, mx, mr)


# --- full-size workloads (sampled heads and rows) -------------------------------

@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_full_size_sampled(name):
    w = W.WORKLOADS[name]
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    qb, kb, vb = W.full_inputs_bits(w)
    step = 7 if w.mode == "structured" else 0
    op, out = _run(w, _dev(qb), _dev(kb), _dev(vb), step=step)
    idx, cnt = op.kv_idx.cpu().numpy(), op.kv_cnt.cpu().numpy()
    rows = sample_rows(w, 40)
    got_all, want_all = [], []
    pinned = total = 0
    for b, h in heads:
        q, k, v, pos = oracle_layout(w, *(W.bits_to_f32(x[b, h]) for x in (qb, kb, vb)))
        if w.mode == "ear":
            _ear_check(op.tables.scores[b, h].cpu().numpy(), q, k, v, w.block, w.scale)
        kept, gate = oracle_kept(w, q, k, step, v=v)
        got = lists_to_sets(idx[b, h], cnt[b, h])
        for i in range(w.nqb):
            total += 1
            if gate[i]:
                pinned += 1
                assert got[i] == kept[i].tolist(), (name, b, h, i)
        want_all.append(O.forward_head(q, k, v, kept, w.block, w.order, w.scale, rows=pos[rows]))
        got_all.append(out[b, h, rows].cpu().numpy())
    assert pinned >= 0.5 * total, (pinned, total)
    mx, mr = err_stats(np.concatenate(got_all), np.concatenate(want_all))
    assert mx <= MAX_ABS and mr <= MEAN_REL, (name, mx, mr)


# --- edge cases -----------------------------------------------------------------

def _rand_bits(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return W.bf16_round(scale * rng.standard_normal(shape).astype(np.float32))[1]


@pytest.mark.parametrize("d,block,order", [(64, 64, 0), (64, 128, 1), (128, 64, 1), (128, 128, 0)])
def test_all_kept_is_dense_attention(d, block, order):
    B, H, N = 1, 2, 700
    qb, kb, vb = (_rand_bits((B, H, N, d), s) for s in (1, 2, 3))
    p = A.Problem(B, H, N, N, d, block, order)
    t = A.allocate_tables(p, "cuda")
    idx = torch.arange(p.nkb, dtype=torch.int32, device="cuda").expand(B, H, p.nqb, p.nkb).contiguous()
    cnt = torch.full((B, H, p.nqb), p.nkb, dtype=torch.int32, device="cuda")
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    A.pool(q_d, k_d, v_d, p, t)
    out = torch.empty(B, H, N, d, device="cuda")
    A.forward(q_d, k_d, v_d, p, t, idx, cnt, out)
    torch.cuda.synchronize()
    rows = np.arange(0, N, 7)
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        want = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(x.astype(np.float64))[None] for x in (q[rows], k, v)))[0].numpy()
        mx, mr = err_stats(out[0, h, rows].cpu().numpy(), want)
        assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)


@pytest.mark.parametrize("order", [0, 1])
def test_nothing_kept_and_bad_list_entries(order):
    """cap 0 (every block compensated) and lists holding out-of-range entries, which
    the forward ignores, against the oracle with nothing kept / the valid entries."""
    B, H, N, d, block = 1, 1, 1000, 128, 128
    qb, kb, vb = _rand_bits((B, H, N, d), 4), _rand_bits((B, H, N, d), 5, 0.3), _rand_bits((B, H, N, d), 6)
    p = A.Problem(B, H, N, N, d, block, order)
    t = A.allocate_tables(p, "cuda")
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    A.pool(q_d, k_d, v_d, p, t)
    q, k, v = (W.bits_to_f32(x[0, 0]) for x in (qb, kb, vb))
    # nothing kept
    idx = torch.zeros(B, H, p.nqb, 1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, H, p.nqb, dtype=torch.int32, device="cuda")
    out = torch.empty(B, H, N, d, device="cuda")
    C.sparse_attn_forward(q_d, k_d, t.v16, t.kbar16, t.vsum16, t.M, idx, cnt, 0, B, H, N, N, d,
                          block, order, 1 / np.sqrt(d), out, C.SA_OUT_F32)
    torch.cuda.synchronize()
    want = O.forward_head(q, k, v, [np.zeros(0, int)] * p.nqb, block, order, 1 / np.sqrt(d))
    mx, mr = err_stats(out[0, 0].cpu().numpy(), want)
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)
    # lists with entries outside [0, nkb) and a count above cap
    lists = [[i, (i + 3) % p.nkb] for i in range(p.nqb)]
    raw = np.full((B, H, p.nqb, 4), -5, np.int32)
    for i, r in enumerate(lists):
        raw[0, 0, i, :3] = [r[0], p.nkb + 2, r[1]]
    idx = torch.from_numpy(raw).cuda()
    cnt = torch.full((B, H, p.nqb), 9, dtype=torch.int32, device="cuda")
    C.sparse_attn_forward(q_d, k_d, t.v16, t.kbar16, t.vsum16, t.M, idx, cnt, 4, B, H, N, N, d,
                          block, order, 1 / np.sqrt(d), out, C.SA_OUT_F32)
    torch.cuda.synchronize()
    want = O.forward_head(q, k, v, [np.array(sorted(r)) for r in lists], block, order, 1 / np.sqrt(d))
    mx, mr = err_stats(out[0, 0].cpu().numpy(), want)
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)


def test_order1_large_queries_keep_the_operand_in_fp16_range():
    """Order 1 forms (scale * alpha) q_t in fp16 with alpha up to 2^11 relative to the row's
    running reference. Queries of magnitude ~600 and keys whose logits rise by ~10.8 (base
    2) from the first centroid tile to the second would put that operand near 2^17; rows
    with such queries rescale earlier, and the output stays finite and matches the oracle."""
    B, H, N, d, block = 1, 2, 8192, 128, 64
    rng = np.random.default_rng(41)
    q = np.empty((B, H, N, d), np.float32)
    k = np.empty((B, H, N, d), np.float32)
    scale = 1 / np.sqrt(d)
    for h in range(H):
        u = rng.choice([-1.0, 1.0], size=d).astype(np.float32)
        q[0, h] = 600.0 * u * (1 + 0.05 * rng.standard_normal((N, 1)).astype(np.float32))
        # logit of a key a * u / d against q = 600 u is scale * 600 * a; base 2: 76.5 a
        a = np.where(np.arange(N) < N // 2, 0.0, 10.8 / (scale * 600 * np.log2(np.e)))
        k[0, h] = (a[:, None] * u[None, :] / d
                   + 1e-4 * rng.standard_normal((N, d))).astype(np.float32)
    qb, kb = W.bf16_round(q)[1], W.bf16_round(k)[1]
    vb = _rand_bits((B, H, N, d), 42)
    p = A.Problem(B, H, N, N, d, block, 1)
    keep = -(-p.nkb // 4)
    kept = {}
    for h in range(H):
        qh, kh = W.bits_to_f32(qb[0, h]), W.bits_to_f32(kb[0, h])
        kept[(0, h)] = O.route_head(qh, kh, block, "topk", scale, keep=keep)[0]
    idx, cnt = _oracle_lists_to_device(W.shrink(W.WORKLOADS["uniform-4k"], B=B, H=H, Nq=N, Nk=N,
                                                d=d, block=block), kept, keep)
    t = A.allocate_tables(p, "cuda")
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    A.pool(q_d, k_d, v_d, p, t)
    out = torch.empty(B, H, N, d, device="cuda")
    A.forward(q_d, k_d, v_d, p, t, idx, cnt, out)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out).all())
    rows = _sample_rows_small(A.Problem(B, H, N, N, d, block, 1), per_tile=1, seed=4)
    got_all, want_all = [], []
    for h in range(H):
        qh, kh, vh = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        want_all.append(O.forward_head(qh, kh, vh, kept[(0, h)], block, 1, scale, rows=rows))
        got_all.append(out[0, h, rows].cpu().numpy())
    mx, mr = err_stats(np.concatenate(got_all), np.concatenate(want_all))
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)


@pytest.mark.parametrize("Nq,Nk,block,order,mode", [
    (1, 5000, 64, 1, "topk"),      # one query row (decode-like), forward split in two
    (2, 1, 128, 0, "topk"),        # a single key
    (63, 63, 64, 2, "topk"),       # one partial block on each side
    (65, 4100, 128, 1, "mass"),    # a full and a one-row query block; ragged keys
    (129, 9000, 64, 0, "mass"),
])
def test_pipeline_tiny_and_ragged_shapes(Nq, Nk, block, order, mode):
    """The whole call (pool, route, forward through BlockSparseAttention, which may split
    the forward) on degenerate shapes, against the oracle's own pipeline."""
    B, H, d = 1, 2, 128
    qb = _rand_bits((B, H, Nq, d), 51)
    kb = _rand_bits((B, H, Nk, d), 52)
    vb = _rand_bits((B, H, Nk, d), 53)
    p = A.Problem(B, H, Nq, Nk, d, block, order)
    op = A.BlockSparseAttention(p, mode, rho=(1, 4), tau=0.9)
    out = op(_dev(qb), _dev(kb), _dev(vb))
    torch.cuda.synchronize()
    op.check()
    scale = 1 / np.sqrt(d)
    got_all, want_all = [], []
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        if mode == "topk":
            kept, sc, counts = O.route_head(q, k, block, "topk", scale, keep=-(-p.nkb // 4))
            gaps, lo, hi = O.gate_diagnostics(sc, counts)
            pinned = gaps > GATE
        else:
            kept, sc, counts = O.route_head(q, k, block, "mass", scale, tau=0.9)
            gaps, lo, hi = O.gate_diagnostics(sc, counts, tau=0.9)
            pinned = (gaps > GATE) & (lo > GATE) & (hi > GATE)
        got = lists_to_sets(op.kv_idx[0, h].cpu().numpy(), op.kv_cnt[0, h].cpu().numpy())
        for i in range(p.nqb):
            if pinned[i]:
                assert got[i] == kept[i].tolist(), (h, i)
        want_all.append(O.forward_head(q, k, v, kept, block, order, scale))
        got_all.append(out[0, h].cpu().numpy())
    mx, mr = err_stats(np.concatenate(got_all), np.concatenate(want_all))
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr, op.last_splits)


@pytest.mark.parametrize("mode,order,block", [
    ("topk", 1, 64), ("topk", 0, 128), ("mass", 1, 128), ("topk_cov", 2, 64), ("topk_cov", 2, 128),
    ("ear", 0, 64),
])
def test_pipeline_head_dim_64(mode, order, block):
    """Every routing mode and order through the d = 64 kernels (pool, route or error-aware
    probe, forward), against the oracle's own pipeline, with ragged ends."""
    B, H, N, d = 1, 2, 3000, 64
    w = W.shrink(W.WORKLOADS["dit-21x30x52"], B=B, H=H, Nq=N, Nk=N, d=d, block=block,
                 order=order, grid=(3, 20, 50))
    qb, kb, vb = W.full_inputs_bits(w)
    p = A.Problem(B, H, N, N, d, block, order)
    rho = (1, 5)
    op = A.BlockSparseAttention(p, mode, rho=rho, tau=0.9)
    out = op(_dev(qb), _dev(kb), _dev(vb))
    torch.cuda.synchronize()
    op.check()
    scale = 1 / np.sqrt(d)
    keep = -(-p.nkb * rho[0] // rho[1])
    got_all, want_all = [], []
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        if mode == "mass":
            kept = O.route_head(q, k, block, "mass", scale, tau=0.9)[0]
        else:
            kept = O.route_head(q, k, block, mode, scale, keep=keep, v=v)[0]
        want_all.append(O.forward_head(q, k, v, kept, block, order, scale))
        got_all.append(out[0, h].cpu().numpy())
    mx, mr = err_stats(np.concatenate(got_all), np.concatenate(want_all))
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mx, mr)


# --- key-range splits of the forward ---------------------------------------------

@pytest.mark.parametrize("Nq,Nk,d,block,order,splits,out_dtype", [
    (300, 20000, 128, 64, 1, 2, torch.float32),    # 313 blocks: 5 runs of 64
    (300, 20000, 128, 64, 1, 3, torch.float32),
    (300, 20000, 128, 64, 0, 5, torch.float32),
    (300, 20000, 128, 64, 1, 9, torch.float32),    # more splits than runs: 4 empty
    (700, 17000, 64, 128, 2, 3, torch.float32),    # 133 blocks, ragged last run
    (260, 30000, 128, 128, 0, 4, torch.bfloat16),  # 235 blocks
    (77, 9000, 64, 64, 1, 16, torch.float32),      # one query tile, ragged everything
])
def test_split_forward_matches_oracle(Nq, Nk, d, block, order, splits, out_dtype):
    """The forward with key-range splits and the merge, on the oracle's top-k lists,
    against the oracle; and against the unsplit forward on the same lists."""
    B, H = 1, 2
    qb = _rand_bits((B, H, Nq, d), 31)
    kb = _rand_bits((B, H, Nk, d), 32, 0.5)
    vb = _rand_bits((B, H, Nk, d), 33)
    p = A.Problem(B, H, Nq, Nk, d, block, order)
    scale = 1 / np.sqrt(d)
    keep = -(-p.nkb // 8)
    kept = {}
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        kept[(0, h)] = O.route_head(q, k, block, "topk", scale, keep=keep)[0]
    idx, cnt = _oracle_lists_to_device(W.shrink(W.WORKLOADS["uniform-4k"], B=B, H=H, Nq=Nq,
                                                Nk=Nk, d=d, block=block), kept, keep)
    t = A.allocate_tables(p, "cuda")
    q_d, k_d, v_d = _dev(qb), _dev(kb), _dev(vb)
    A.pool(q_d, k_d, v_d, p, t)
    work = torch.empty(C.sparse_attn_forward_work_bytes(B, H, Nq, d, splits) // 4, device="cuda")
    out = torch.empty(B, H, Nq, d, dtype=out_dtype, device="cuda")
    ref = torch.empty(B, H, Nq, d, dtype=out_dtype, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.forward(q_d, k_d, v_d, p, t, idx, cnt, out, err_flag=flag, splits=splits, work=work)
    A.forward(q_d, k_d, v_d, p, t, idx, cnt, ref, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    got_all, want_all = [], []
    for h in range(H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        want_all.append(O.forward_head(q, k, v, kept[(0, h)], block, order, scale))
        got_all.append(out[0, h].float().cpu().numpy())
    got, want = np.concatenate(got_all), np.concatenate(want_all)
    mx, mr = err_stats(got, want)
    floor = 0.0
    if out_dtype == torch.bfloat16:
        floor = err_stats(torch.from_numpy(want).to(torch.bfloat16).double().numpy(), want)[1]
    assert mx <= MAX_ABS and mr <= MEAN_REL + floor, (mx, mr, floor)
    # the split only reorders fp32 sums and moves the fp16 rounding of P with the
    # running maxima: far below the oracle tolerance
    d_ab = (out.float() - ref.float()).abs().max().item()
    assert d_ab <= (2e-3 if out_dtype == torch.float32 else 2e-2), d_ab


def test_split_plan_and_work_bytes():
    """The library's split choice: none for grids of many waves, some for the world-model
    chunk, never more than the 64-block runs; scratch size as documented."""
    for (B, H, Nq, Nk, d, block) in [(1, 40, 75600, 75600, 128, 128), (1, 24, 32760, 32760, 128, 128)]:
        assert C.sparse_attn_forward_split_plan(B, H, Nq, Nk, d, block) == (1, 0)
    n, b = C.sparse_attn_forward_split_plan(4, 16, 1560, 63960, 128, 64)
    assert 2 <= n <= 16 and b == n * 4 * 16 * 1560 * 130 * 4
    n, _ = C.sparse_attn_forward_split_plan(1, 1, 1560, 4096, 128, 64)
    assert n == 1  # a single run of 64 blocks cannot be split
    assert C.sparse_attn_forward_work_bytes(2, 3, 100, 64, 1) == 0
    assert C.sparse_attn_forward_work_bytes(2, 3, 100, 64, 4) == 4 * 2 * 3 * 100 * 66 * 4


def test_split_forward_empty_and_invalid():
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    i = torch.zeros(4, dtype=torch.int32, device="cuda")
    # no queries: nothing to do, even without scratch
    C.sparse_attn_forward_split(x, x, x, x, x, x, i, i, 1, 1, 1, 0, 100, 128, 128, 1, 0.1, 4,
                                None, f, 0)
    with pytest.raises(C.SparseAttnError):  # scratch missing
        C.sparse_attn_forward_split(x, x, x, x, x, x, i, i, 1, 1, 1, 64, 64, 64, 64, 0, 0.1, 2,
                                    None, f, 0)
    with pytest.raises(C.SparseAttnError):  # too many splits
        C.sparse_attn_forward_split(x, x, x, x, x, x, i, i, 1, 1, 1, 64, 64, 64, 64, 0, 0.1, 17,
                                    f, f, 0)


@pytest.mark.parametrize("order", [0, 1])
def test_incremental_pool_equals_full_pool(order):
    """A KV cache whose last blocks change: pooling only those blocks over the tables of
    the old cache gives the tables of a full pool of the new cache, bit for bit."""
    B, H, d, block, Nk, Nq = 1, 2, 128, 64, 64 * 40 + 24, 300
    j0 = 33
    qb = _rand_bits((B, H, Nq, d), 50)
    kb1, vb1 = _rand_bits((B, H, Nk, d), 51), _rand_bits((B, H, Nk, d), 52)
    kb2, vb2 = kb1.copy(), vb1.copy()
    kb2[:, :, j0 * block:] = _rand_bits((B, H, Nk - j0 * block, d), 53)
    vb2[:, :, j0 * block:] = _rand_bits((B, H, Nk - j0 * block, d), 54)
    p = A.Problem(B, H, Nq, Nk, d, block, order)
    t_inc, t_full = A.allocate_tables(p, "cuda"), A.allocate_tables(p, "cuda")
    q = _dev(qb)
    A.pool(q, _dev(kb1), _dev(vb1), p, t_inc)
    A.pool(q, _dev(kb2), _dev(vb2), p, t_inc, kv_block_start=j0)
    A.pool(q, _dev(kb2), _dev(vb2), p, t_full)
    torch.cuda.synchronize()
    for name in ("qbar", "kbar_t", "vsum", "kbar16", "vsum16", "M", "v16"):
        a, b = getattr(t_inc, name), getattr(t_full, name)
        if a is not None:
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name


def test_empty_problems_are_no_ops():
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    i = torch.zeros(16, dtype=torch.int32, device="cuda")
    C.sparse_attn_pool(x, x, x, 0, 4, 100, 100, 128, 128, 1, f, f, f, x, x, x, x)
    C.sparse_attn_route(f, f, 1, 1, 0, 10, 128, 0, 1, 4, 0.9, 0.1, i, i, 3)
    C.sparse_attn_structured_mask(1, 1, 0, 100, 64, 10, 10, 1, 1, 1, 0, 0, i, i, 2)
    C.sparse_attn_forward(x, x, x, x, x, x, i, i, 1, 1, 1, 0, 100, 128, 128, 1, 0.1, f, 0)
    torch.cuda.synchronize()
    assert int(i.abs().sum()) == 0


def test_invalid_arguments_raise():
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(64, dtype=torch.float32, device="cuda")
    i = torch.zeros(64, dtype=torch.int32, device="cuda")
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_forward(x, x, x, x, x, x, i, i, 1, 1, 1, 64, 64, 96, 64, 0, 0.1, f, 0)
    assert e.value.code == C.SA_ERR_INVALID and "d must be" in str(e.value)
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_forward(x.data_ptr() + 2, x, x, x, x, x, i, i, 1, 1, 1, 64, 64, 64, 64, 0,
                              0.1, f, 0)
    assert e.value.code == C.SA_ERR_INVALID and "aligned" in str(e.value)
    with pytest.raises(C.SparseAttnError) as e:   # cap below the keep count
        C.sparse_attn_route(f, f, 1, 1, 4, 10, 64, 0, 1, 2, 0.9, 0.1, i, i, 4)
    assert e.value.code == C.SA_ERR_INVALID
    with pytest.raises(C.SparseAttnError) as e:   # mass routing needs cap >= nkb
        C.sparse_attn_route(f, f, 1, 1, 4, 10, 64, 1, 1, 2, 0.9, 0.1, i, i, 9)
    assert e.value.code == C.SA_ERR_INVALID
    with pytest.raises(C.SparseAttnError):        # order 1 without M
        C.sparse_attn_pool(x, x, x, 1, 1, 64, 64, 64, 64, 1, f, f, f, x, x, None, x)


def test_bounded_wait_gives_up_and_reports(small_inputs):
    """A wait on an mbarrier that nothing completes ends after its bounded rounds, sets
    the error word and returns; the context stays usable for a real call afterwards."""
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    C.sparse_attn_wait_selftest(flag, 256, waited)
    torch.cuda.synchronize()
    assert int(waited.item()) == 0 and int(flag.item()) & 1
    w, qb, kb, vb = small_inputs("uniform-4k")
    op, out = _run(w, _dev(qb), _dev(kb), _dev(vb))
    assert int(op.err_flag.item()) == 0 and torch.isfinite(out).all()
    with pytest.raises(C.SparseAttnError) as e:   # the host helper turns a set flag into an error
        op.err_flag.fill_(1)
        op.check()
    assert e.value.code == C.SA_ERR_TIMEOUT


@pytest.mark.parametrize("name", ["dit-small", "kmeans-small", "longvideo-small", "worldmodel-small",
                                  "ear-small", "hybrid-small"])
def test_host_call_equals_device_call(name, small_inputs):
    """run_from_host (head ranges, copies overlapped with the compute) gives the device
    call's output bit for bit (the forward's split count is the whole problem's)."""
    w, qb, kb, vb = small_inputs(name)
    if name in ("dit-small", "kmeans-small"):   # enough heads for several ranges of four
        w = W.shrink(w, H=12, Nq=3000, Nk=3000, grid=(3, 20, 50))
        qb, kb, vb = W.full_inputs_bits(w)
    if name == "worldmodel-small":  # ranges of four heads, forward split in two
        w = W.shrink(w, H=8)
        qb, kb, vb = W.full_inputs_bits(w)
    step = w.steps[-1] if w.mode == "structured" else 0
    op, out = _run(w, _dev(qb), _dev(kb), _dev(vb), step=step)
    want = out.clone()
    pin = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_h = torch.empty(want.shape, dtype=want.dtype, pin_memory=True)
    for chunks in (1, 3, 8):
        out_h.zero_()
        op.run_from_host(pin(qb), pin(kb), pin(vb), out_h, step=step, chunks=chunks)
        torch.cuda.synchronize()
        op.check()
        assert torch.equal(out_h, want.cpu()), chunks


@pytest.mark.parametrize("name", ["dit-small", "ear-small", "kmeans-small", "hybrid-small",
                                  "longvideo-small"])
def test_graph_replay_equals_eager_call(name, small_inputs):
    """A captured call replays the same launches: equal output, also after the inputs
    change in place."""
    w, qb, kb, vb = small_inputs(name)
    step = w.steps[-1] if w.mode == "structured" else 0
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    op, out = _run(w, q, k, v, step=step)
    want = out.clone()
    g = op.capture(q, k, v, step=step)
    op.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(op.out, want)
    k.copy_(torch.roll(k, 7, dims=2))               # new keys, same buffers
    _, want2 = _run(w, q, k, v, step=step)
    want2 = want2.clone()
    op.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    op.check()
    assert torch.equal(op.out, want2)
    del g


@pytest.mark.parametrize("name", ["dit-small", "ear-small", "kmeans-small", "hybrid-small",
                                  "worldmodel-small"])
def test_repeat_calls_are_bitwise_deterministic(name, small_inputs):
    w, qb, kb, vb = small_inputs(name)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    op, a = _run(w, q, k, v)
    a = a.clone()
    extra = [op.tables.scores.clone()] if w.mode == "ear" else []
    if w.clusters:
        extra += [op.cl_q.perm.clone(), op.cl_k.centroids.clone()]
    _, b = _run(w, q, k, v)
    assert torch.equal(a, b)
    op2, _ = _run(w, q, k, v)
    if w.mode == "ear":
        assert torch.equal(op2.tables.scores, extra[0])
    if w.clusters:
        assert torch.equal(op2.cl_q.perm, extra[-2]) and torch.equal(op2.cl_k.centroids, extra[-1])


@pytest.mark.parametrize("mode", ["topk", "mass"])
def test_route_exact_ties_break_by_lower_index(mode):
    """Key blocks duplicated pairwise give bit-identical centroids, hence exactly tied
    scores on both sides; the kept sets must then match the oracle on every row,
    including rows whose cutoff falls inside a tie."""
    B, H, d, block, nkb = 1, 2, 64, 64, 40
    N = nkb * block
    rng = np.random.default_rng(7)
    kb = np.empty((B, H, N, d), np.uint16)
    for h in range(H):
        base = rng.standard_normal((nkb // 2, block, d)).astype(np.float32)
        blocks = np.repeat(base, 2, axis=0)          # block 2m and 2m+1 identical
        kb[0, h] = W.bf16_round(blocks.reshape(N, d))[1]
    qb = _rand_bits((B, H, N, d), 8)
    vb = _rand_bits((B, H, N, d), 9)
    w = W.Workload(name="ties", B=B, H=H, Nq=N, Nk=N, d=d, block=block, order=0, mode=mode,
                   rho=(7, 40), tau=0.6)
    op, _ = _run(w, _dev(qb), _dev(kb), _dev(vb))
    idx, cnt = op.kv_idx.cpu().numpy(), op.kv_cnt.cpu().numpy()
    for h in range(H):
        q, k = W.bits_to_f32(qb[0, h]), W.bits_to_f32(kb[0, h])
        if mode == "topk":
            kept = O.route_head(q, k, block, "topk", w.scale, keep=w.keep())[0]
        else:
            kept = O.route_head(q, k, block, "mass", w.scale, tau=w.tau)[0]
        got = lists_to_sets(idx[0, h], cnt[0, h])
        assert got == [x.tolist() for x in kept], (mode, h)
