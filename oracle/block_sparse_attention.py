"""fp64 CPU oracle for block-sparse attention with skipped-block compensation.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain definition that the
CUDA path is checked against. Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it; the library never does, and it
imports nothing from the library.

Every function works on ONE (batch, head) pair in float64. Inputs are the
bf16-rounded Q, K, V converted exactly to float64.

Sources (page title, section):
  [PISA]  "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
          Transformers", §2 "Méthodologie": "Cohérence de Normalisation",
          "Algorithme Central" (o_t = N_t / D_t, the numerator N_t and
          alpha_{t,j} = exp(q_t kbar_j^T)), "Implémentation Matérielle"
          (pre-computation; phases 1-3).
  [LVSA]  "LVSA: Training-Free Sparse Attention for Long Video Diffusion",
          §2 "Mécanisme Central" (A(t) = G u W(t); rotating anchors G_s shifted
          by s mod T_per; local window W(t)).
  [EAR]   "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video
          Generation via Error-aware Routing", §2 A-B (centroid substitution;
          query centroids as proxies for a block's queries).

Readings where the pages are silent (each is listed with its reason in the
design notes):
  * the 1/sqrt(d) scale multiplies every logit, the routing scores and the
    first-order term (the PISA numerator is printed without it);
  * the first-order term is per block, M_j = sum_r (k_r - kbar_j) v_r^T, and
    enters the numerator only: its denominator share sums to zero because
    sum_r (k_r - kbar_j) = 0;
  * a partial last block uses its true token count n_j for means and for the
    order-0 denominator;
  * top-rho keeps ceil(rho * nkb) blocks (integer arithmetic); order is
    (score descending, block index ascending);
  * mass-tau keeps the shortest such prefix whose softmax mass reaches tau
    (cumulative >= tau);
  * structured mode: anchors G_s = {(s mod T_per) + T_per * m}, window
    [t - W, t + W] clipped to the video; a KV block is kept for a query block
    when any (query token, key token) pair of the two blocks is allowed; with a
    budget C (LVSA extended adaptive windows) the window grows one frame at a
    time, alternately after and before it, until |A(t)| reaches C;
  * hybrid order (order 2, PISA "Algorithme Central", global first-order
    correction): Hbar is the plain mean of the per-block matrices M_j over all
    blocks of the head, and the numerator gains scale * q_t Hbar * sum_j alpha_tj
    over the skipped blocks (no denominator term, as for order 1);
  * error-aware routing (EAR §2 B): with the query centroid qbar_i as the proxy
    query, the error of block j is err_ij = || sum_r (exp(s_r) - exp(s_c)) v_r ||^2
    with s_r = scale qbar_i.k_r and s_c = scale qbar_i.kbar_j: the squared error
    of the centroid substitution (order 0) on the block's share of the unnormalised
    attention numerator. The score is ln(err_ij / n_j) (error per unit of cost, the
    cost being the block's token count; the log only changes the scale), blocks are
    ranked by it, ties by index, and the top ceil(rho nkb) are kept (the greedy
    selection under a density budget, with the budget read as a block count);
  * covariance-aware top-k (PISA "Routage Sensible a la Covariance"): the
    norm ||H_j - Hbar||_2 is read as the 2-norm of the matrix entries
    (Frobenius), and the selection score is s_ij + ln ||H_j - Hbar||, the log of
    the first-order error bound alpha_ij * scale * |qbar_i| * ||H_j - Hbar||
    up to a term that is the same for every block of the row.
"""
from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# Blocking
# ---------------------------------------------------------------------------

def block_ranges(n_tokens: int, block: int):
    """Token ranges [start, end) of the blocks of b tokens; the last may be partial."""
    return [(s, min(s + block, n_tokens)) for s in range(0, n_tokens, block)]


# ---------------------------------------------------------------------------
# Pooling  [PISA §2 "Implémentation Matérielle": pre-computation of block
# centroids and value sums; "Algorithme Central": kbar_j and sum_n v_{j,n}]
# ---------------------------------------------------------------------------

def pool_queries(q: np.ndarray, block: int) -> np.ndarray:
    """qbar_i = mean of the query rows of block i  [EAR §2 B: query centroids as proxies]."""
    q = np.asarray(q, dtype=np.float64)
    return np.stack([q[s:e].mean(axis=0) for s, e in block_ranges(q.shape[0], block)])


def pool_keys_values(k: np.ndarray, v: np.ndarray, block: int, order: int):
    """Per KV block j: centroid kbar_j, value sum S_j, token count n_j and (order 1 or 2) M_j.

    M_j[a, c] = sum over tokens r of block j of (k_r[a] - kbar_j[a]) * v_r[c]:
    the first-order Taylor matrix of the block (key dim a, value dim c).
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kbar, vsum, counts, mats = [], [], [], []
    for s, e in block_ranges(k.shape[0], block):
        kj, vj = k[s:e], v[s:e]
        kb = kj.mean(axis=0)
        kbar.append(kb)
        vsum.append(vj.sum(axis=0))
        counts.append(e - s)
        if order >= 1:
            mats.append((kj - kb).T @ vj)
    m = np.stack(mats) if order >= 1 else None
    return np.stack(kbar), np.stack(vsum), np.asarray(counts, dtype=np.int64), m


def global_first_order(mats: np.ndarray) -> np.ndarray:
    """Hbar = mean over all blocks of the per-block first-order matrices M_j
    [PISA §2 "Algorithme Central": global first-order statistic]."""
    return np.asarray(mats, np.float64).mean(axis=0)


def covariance_norms(mats: np.ndarray, hbar: np.ndarray) -> np.ndarray:
    """||M_j - Hbar|| per block, as the 2-norm of the matrix entries
    [PISA §2 "Routage Sensible a la Covariance"]."""
    diff = np.asarray(mats, np.float64) - np.asarray(hbar, np.float64)[None]
    return np.sqrt((diff * diff).sum(axis=(1, 2)))


# ---------------------------------------------------------------------------
# Routing  [PISA §2 top-k selection of critical blocks S_i; EAR §2 B query
# centroids; keep rules as stated in the module docstring]
# ---------------------------------------------------------------------------

def routing_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Pooled logits s_ij = scale * qbar_i . kbar_j."""
    return scale * (np.asarray(qbar, np.float64) @ np.asarray(kbar, np.float64).T)


def keep_count(nkb: int, rho_num: int, rho_den: int) -> int:
    """ceil(rho * nkb) for rho = rho_num / rho_den, in integer arithmetic."""
    return -(-rho_num * nkb // rho_den)


def block_order(scores_row: np.ndarray) -> np.ndarray:
    """Block indices sorted by (score descending, index ascending)."""
    j = np.arange(scores_row.shape[0])
    return np.lexsort((j, -scores_row))


def route_topk(scores: np.ndarray, keep: int):
    """Kept block indices (ascending) of each query block under top-k."""
    return [np.sort(block_order(row)[:keep]) for row in scores]


def row_softmax(scores_row: np.ndarray) -> np.ndarray:
    """softmax over KV blocks, with max subtraction."""
    z = np.exp(scores_row - scores_row.max())
    return z / z.sum()


def route_mass(scores: np.ndarray, tau: float):
    """Kept blocks of each query block: the shortest prefix of the block order whose
    softmax mass reaches tau. Returns (kept lists, prefix lengths)."""
    kept, counts = [], []
    for row in scores:
        order = block_order(row)
        cum = np.cumsum(row_softmax(row)[order])
        k = int(np.searchsorted(cum, tau, side="left")) + 1
        k = min(k, row.shape[0])
        kept.append(np.sort(order[:k]))
        counts.append(k)
    return kept, counts


def gate_diagnostics(scores: np.ndarray, counts, tau=None):
    """Per query block: the logit gap at the cutoff, s_(k) - s_(k+1), and for mass
    routing the two margins tau - C_(k-1) and C_k - tau (inf where undefined)."""
    gaps, lo, hi = [], [], []
    for row, k in zip(scores, counts):
        order = block_order(row)
        s_sorted = row[order]
        gaps.append(s_sorted[k - 1] - s_sorted[k] if 0 < k < row.shape[0] else math.inf)
        if tau is not None:
            cum = np.cumsum(row_softmax(row)[order])
            lo.append(tau - cum[k - 2] if k >= 2 else math.inf)
            hi.append(cum[k - 1] - tau)
    return np.asarray(gaps), np.asarray(lo), np.asarray(hi)


# ---------------------------------------------------------------------------
# Structured mask  [LVSA §2 "Mécanisme Central"]
# ---------------------------------------------------------------------------

def anchor_frames(step: int, period: int, n_anchors: int, n_frames: int):
    """G_s: n_anchors frames spaced by T_per, shifted by s mod T_per."""
    base = step % period
    return {base + period * m for m in range(n_anchors) if base + period * m < n_frames}


def attend_frames(t: int, step: int, window: int, period: int, n_anchors: int, n_frames: int,
                  budget: int = 0):
    """A(t) = G_s u W(t), with W(t) = {t - window, ..., t + window} inside the video.

    budget C > 0 [LVSA §2 "Fenêtres Adaptatives Étendues"]: while |G_s u W(t)| < C and
    W(t) is not the whole video, the window grows by one frame, alternately after and
    before it (skipping a side that has reached the edge), so that overlaps with the
    anchors and clipping at the edges are made up: |A(t)| = max(|G_s u W(t)|, min(C, T)).
    """
    anchors = anchor_frames(step, period, n_anchors, n_frames)
    lo, hi = max(0, t - window), min(n_frames - 1, t + window)
    after = True
    while budget > 0 and len(anchors | set(range(lo, hi + 1))) < budget and (lo > 0 or hi < n_frames - 1):
        if (after and hi < n_frames - 1) or lo == 0:
            hi += 1
        else:
            lo -= 1
        after = not after
    return anchors | set(range(lo, hi + 1))


def structured_kept(Nq: int, Nk: int, block: int, frame_tokens: int, n_frames: int,
                    window: int, n_anchors: int, period: int, step: int, q_frame0: int = 0,
                    budget: int = 0):
    """Kept KV blocks per query block: block j is kept for query block i when some
    query token of i and some key token of j lie in frames (tq, tk) with tk in A(tq)."""
    key_frames = [{r // frame_tokens for r in range(ks, ke)} for ks, ke in block_ranges(Nk, block)]
    kept = []
    for qs, qe in block_ranges(Nq, block):
        q_frames = sorted({(q_frame0 * frame_tokens + t) // frame_tokens for t in range(qs, qe)})
        allowed = set()
        for t in q_frames:
            allowed |= attend_frames(t, step, window, period, n_anchors, n_frames, budget)
        row = [j for j, kf in enumerate(key_frames) if kf & allowed]
        kept.append(np.asarray(row, dtype=np.int64))
    return kept


# ---------------------------------------------------------------------------
# Forward  [PISA §2 "Algorithme Central" and "Cohérence de Normalisation":
# exact terms for kept blocks; order-0 term alpha_{t,j} * S_j; first-order
# term; both inside the numerator and the denominator of one softmax]
# ---------------------------------------------------------------------------

def forward_rows(q_rows: np.ndarray, row_qblock, k: np.ndarray, v: np.ndarray,
                 kbar: np.ndarray, vsum: np.ndarray, counts: np.ndarray, mats,
                 kept, block: int, order: int, scale: float, hbar=None) -> np.ndarray:
    """Output rows o_t = N_t / D_t for the query rows q_rows.

    row_qblock[t] is the query block of row t; kept[i] lists the kept KV blocks
    of query block i. For row t:
      exact logits    l_r  = scale * q_t . k_r        for tokens r of kept blocks
      centroid logits c_j  = scale * q_t . kbar_j     for skipped blocks j
      m = max of all of them
      N_t = sum_r e^(l_r - m) v_r
            + sum_j e^(c_j - m) (S_j + [order 1] scale * q_t M_j
                                     + [order 2] scale * q_t Hbar)
      D_t = sum_r e^(l_r - m) + sum_j e^(c_j - m) n_j
    Order 2 (hybrid) needs ``hbar``, the mean of the per-block M_j.
    """
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nkb = kbar.shape[0]
    ranges = block_ranges(k.shape[0], block)
    out = np.empty((q_rows.shape[0], v.shape[1]))
    for t, (qt, i) in enumerate(zip(np.asarray(q_rows, np.float64), row_qblock)):
        kept_set = set(int(j) for j in kept[i])
        skipped = [j for j in range(nkb) if j not in kept_set]
        tok = np.concatenate([np.arange(*ranges[j]) for j in sorted(kept_set)]) if kept_set \
            else np.zeros(0, dtype=np.int64)
        l = scale * (k[tok] @ qt)
        c = scale * (kbar[skipped] @ qt) if skipped else np.zeros(0)
        m = max(l.max(initial=-math.inf), c.max(initial=-math.inf))
        we = np.exp(l - m)
        wc = np.exp(c - m)
        num = we @ v[tok]
        den = we.sum()
        for w, j in zip(wc, skipped):
            term = vsum[j].copy()
            if order == 1:
                term += scale * (qt @ mats[j])
            num += w * term
            den += w * counts[j]
        if order == 2 and skipped:
            num += scale * wc.sum() * (qt @ hbar)
        out[t] = num / den
    return out


def forward_head(q, k, v, kept, block: int, order: int, scale: float, rows=None):
    """Pool K/V and run :func:`forward_rows` on all rows of a head, or on ``rows``."""
    kbar, vsum, counts, mats = pool_keys_values(k, v, block, 1 if order == 2 else order)
    hbar = global_first_order(mats) if order == 2 else None
    q = np.asarray(q, np.float64)
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    return forward_rows(q[rows], rows // block, k, v, kbar, vsum, counts, mats,
                        kept, block, order, scale, hbar=hbar)


def covariance_scores(scores: np.ndarray, cnorms: np.ndarray) -> np.ndarray:
    """Covariance-aware selection scores s_ij + ln ||M_j - Hbar||
    [PISA §2 "Routage Sensible a la Covariance"]."""
    with np.errstate(divide="ignore"):
        return np.asarray(scores, np.float64) + np.log(np.asarray(cnorms, np.float64))[None, :]


def ear_scores(qbar: np.ndarray, k: np.ndarray, v: np.ndarray, block: int, scale: float):
    """Error-aware routing scores ln(err_ij / n_j)  [EAR §2 B: the squared error of the
    centroid approximation per block, query centroids as proxies, error per unit of
    cost]. err_ij = 0 (a block whose keys all give the same logit) scores -inf.

    Every weight of row i and block j is taken relative to m = the largest exact logit
    of the block: err = exp(2 m) * || sum_r (exp(s_r - m) - exp(s_c - m)) v_r ||^2.
    """
    qbar = np.asarray(qbar, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    kbar, _, counts, _ = pool_keys_values(k, v, block, 0)
    out = np.empty((qbar.shape[0], kbar.shape[0]))
    for j, (s, e) in enumerate(block_ranges(k.shape[0], block)):
        logit = scale * (qbar @ k[s:e].T)                 # exact logits s_r, [nqb, n_j]
        cen = scale * (qbar @ kbar[j])                    # centroid logit s_c
        m = logit.max(axis=1)
        x = (np.exp(logit - m[:, None]) - np.exp(cen - m)[:, None]) @ v[s:e]
        err = (x * x).sum(axis=1)
        with np.errstate(divide="ignore"):
            out[:, j] = np.log(err) + 2.0 * m - np.log(counts[j])
    return out


def route_head(q, k, block: int, mode: str, scale: float, keep=None, tau=None, v=None):
    """Pooled routing for one head. Returns (kept lists, scores, prefix lengths).

    modes "topk_cov" and "ear" need ``v`` (the per-block M_j; the numerator errors)
    and return their own scores."""
    qbar = pool_queries(q, block)
    if mode == "ear":
        s = ear_scores(qbar, k, v, block, scale)
        return route_topk(s, keep), s, [keep] * s.shape[0]
    if mode == "topk_cov":
        kbar, _, _, mats = pool_keys_values(k, v, block, 1)
        s = covariance_scores(routing_scores(qbar, kbar, scale),
                              covariance_norms(mats, global_first_order(mats)))
        return route_topk(s, keep), s, [keep] * s.shape[0]
    kbar = pool_keys_values(k, np.zeros((k.shape[0], 1)), block, 0)[0]
    s = routing_scores(qbar, kbar, scale)
    if mode == "topk":
        return route_topk(s, keep), s, [keep] * s.shape[0]
    if mode == "mass":
        kept, counts = route_mass(s, tau)
        return kept, s, counts
    raise ValueError(mode)


# ---------------------------------------------------------------------------
# Independent twin: per-pair weights, no pooled tables
# ---------------------------------------------------------------------------

def brute_force_pairs(q, k, v, kept, block: int, order: int, scale: float) -> np.ndarray:
    """Same output as the blockwise forward, built pair by pair with plain loops.

    Weight of query t on key r of block j (relative to a per-row shift m):
      kept j:            e^(scale q.k_r - m)
      skipped, order 0:  e^(scale q.kbar_j - m)
      skipped, order 1:  e^(scale q.kbar_j - m) * (1 + scale q.(k_r - kbar_j))
    and o_t = sum_r w_tr v_r / sum_r w_tr. The first-order factor is the Taylor
    expansion of e^(scale q.k_r) about kbar_j. Loops are over pairs, so keep N
    small (a few hundred).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, nk = q.shape[0], k.shape[0]
    out = np.empty((nq, v.shape[1]))
    for t in range(nq):
        i = t // block
        kept_set = set(int(j) for j in kept[i])
        logit = np.empty(nk)
        lin = np.ones(nk)
        for r in range(nk):
            j = r // block
            js, je = j * block, min((j + 1) * block, nk)
            if j in kept_set:
                logit[r] = scale * float(np.dot(q[t], k[r]))
            else:
                centroid = k[js:je].sum(axis=0) / (je - js)
                logit[r] = scale * float(np.dot(q[t], centroid))
                if order == 1:
                    lin[r] = 1.0 + scale * float(np.dot(q[t], k[r] - centroid))
        w = np.exp(logit - logit.max()) * lin
        out[t] = (w @ v) / w.sum()
    return out


def dense_attention_loops(q, k, v, scale: float) -> np.ndarray:
    """softmax(scale q k^T) v with explicit loops over rows and keys (tiny inputs)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.empty((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        logits = [scale * sum(float(a) * float(b) for a, b in zip(q[t], k[r])) for r in range(k.shape[0])]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        out[t] = sum(wr * v[r] for wr, r in zip(w, range(k.shape[0]))) / z
    return out
