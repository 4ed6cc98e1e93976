"""Torch-side plumbing around the C ABI: table and list allocation, and the
three-stage call (pool -> route or structured mask -> forward) on one stream.

Torch only provides device memory and the stream; each stage is one call into
``libsparse_attn.so``.
"""
from __future__ import annotations

import dataclasses
import functools
import math
from typing import Optional

import torch

from . import sparse_attn as C
from . import sparse_attn as _C


@dataclasses.dataclass
class Tables:
    """Pooled tables of one problem (layouts as in include/sparse_attn.h)."""
    qbar: torch.Tensor      # [B,H,nqb,d] fp32
    kbar_t: torch.Tensor    # [B,H,d,nkb] fp32
    vsum: torch.Tensor      # [B,H,nkb,d] fp32
    kbar16: torch.Tensor    # [B,H,2,nkb,d] bf16: centroid hi and lo parts
    vsum16: torch.Tensor    # [B,H,nkb,d] fp16
    M: Optional[torch.Tensor]  # [B,H,nkb,d,d] fp16 (order 1 or 2)
    v16: torch.Tensor       # [B,H,Nk,d] fp16 copy of V
    hbar: Optional[torch.Tensor] = None    # [B,H,d,d] fp32 global first-order matrix (order 2)
    hbar16: Optional[torch.Tensor] = None  # [B,H,d,d] fp16
    cov: Optional[torch.Tensor] = None     # [B,H,nkb] fp32 ||M_j - Hbar|| (order 2)
    scores: Optional[torch.Tensor] = None  # [B,H,nqb,nkb] fp32 error-aware routing scores


@dataclasses.dataclass
class Problem:
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    block: int
    order: int  # 0, 1 (first-order term per block) or 2 (global first-order term)

    @property
    def nqb(self) -> int:
        return -(-self.Nq // self.block)

    @property
    def nkb(self) -> int:
        return -(-self.Nk // self.block)


def allocate_tables(p: Problem, device, ear: bool = False) -> Tables:
    f32 = dict(dtype=torch.float32, device=device)
    h16 = dict(dtype=torch.float16, device=device)
    return Tables(
        qbar=torch.empty(p.B, p.H, p.nqb, p.d, **f32),
        kbar_t=torch.empty(p.B, p.H, p.d, p.nkb, **f32),
        vsum=torch.empty(p.B, p.H, p.nkb, p.d, **f32),
        kbar16=torch.empty(p.B, p.H, 2, p.nkb, p.d, dtype=torch.bfloat16, device=device),
        vsum16=torch.empty(p.B, p.H, p.nkb, p.d, **h16),
        M=torch.empty(p.B, p.H, p.nkb, p.d, p.d, **h16) if p.order >= 1 else None,
        v16=torch.empty(p.B, p.H, p.Nk, p.d, **h16),
        hbar=torch.empty(p.B, p.H, p.d, p.d, **f32) if p.order == 2 else None,
        hbar16=torch.empty(p.B, p.H, p.d, p.d, **h16) if p.order == 2 else None,
        cov=torch.empty(p.B, p.H, p.nkb, **f32) if p.order == 2 else None,
        scores=torch.empty(p.B, p.H, p.nqb, p.nkb, **f32) if ear else None,
    )


@dataclasses.dataclass
class Clustering:
    """Buffers of one tensor's k-means and its group-major layout (include/sparse_attn.h)."""
    C: int
    iters: int
    centroids: torch.Tensor  # [B,H,C,d] fp64
    cwork: torch.Tensor      # scratch bytes
    iwork: torch.Tensor      # scratch int32
    labels: torch.Tensor     # [B,H,N] int32
    perm: torch.Tensor       # [B,H,N] int32: perm[p] = original index at position p
    offsets: torch.Tensor    # [B,H,C+1] int32


def allocate_clustering(B, H, N, d, C, iters, device) -> Clustering:
    _, s_cw, s_iw = _C.sparse_attn_kmeans_sizes(B, H, N, d, C)
    i32 = dict(dtype=torch.int32, device=device)
    return Clustering(
        C=C, iters=iters,
        centroids=torch.empty(B, H, C, d, dtype=torch.float64, device=device),
        cwork=torch.empty(max(s_cw, 16), dtype=torch.uint8, device=device),
        iwork=torch.empty(max(s_iw // 4, 4), **i32),
        labels=torch.empty(B, H, N, **i32), perm=torch.empty(B, H, N, **i32),
        offsets=torch.empty(B, H, C + 1, **i32))


def kmeans(x, cl: Clustering, err_flag=None, stream=None):
    """k-means of x's rows per (b, h) and the stable group-major order of the labels."""
    B, H, N, d = x.shape
    _C.sparse_attn_kmeans(x, B, H, N, d, cl.C, cl.iters, cl.centroids, cl.cwork, cl.iwork,
                          cl.labels, cl.perm, cl.offsets, err_flag, stream)


def permute_rows(src, perm, dst, gather=True, stream=None):
    """gather: dst[p] = src[perm[p]]; otherwise dst[perm[p]] = src[p] (per (b, h))."""
    B, H, N, d = src.shape
    _C.sparse_attn_permute_rows(src, perm, B, H, N, d * src.element_size(), gather, dst, stream)


def allocate_lists(p: Problem, cap: int, device):
    return (torch.zeros(p.B, p.H, p.nqb, max(cap, 1), dtype=torch.int32, device=device),
            torch.zeros(p.B, p.H, p.nqb, dtype=torch.int32, device=device))


def _check_inputs(q, k, v):
    for name, x in (("q", q), ("k", k), ("v", v)):
        if not (x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 4):
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor [B,H,N,d]")


def pool(q, k, v, p: Problem, t: Tables, stream=None, kv_block_start: int = 0, err_flag=None):
    """Pooled tables; with order 2 also the global first-order matrix and the
    per-block covariance norms. kv_block_start > 0 pools only the KV blocks from there
    on (a growing KV cache whose earlier blocks were pooled by an earlier call).
    err_flag (device int32) receives SA_FLAG_RANGE if an fp16 table value overflows."""
    if kv_block_start:
        C.sparse_attn_pool_incremental(q, k, v, p.B, p.H, p.Nq, p.Nk, p.d, p.block, p.order,
                                       kv_block_start, t.qbar, t.kbar_t, t.vsum, t.kbar16,
                                       t.vsum16, t.M, t.v16, err_flag, stream)
    else:
        C.sparse_attn_pool(q, k, v, p.B, p.H, p.Nq, p.Nk, p.d, p.block, p.order, t.qbar,
                           t.kbar_t, t.vsum, t.kbar16, t.vsum16, t.M, t.v16, err_flag, stream)
    if p.order == 2:
        C.sparse_attn_hbar(t.M, p.B, p.H, p.nkb, p.d, t.hbar, t.hbar16, t.cov, stream)


def ear_scores(k, v, p: Problem, t: Tables, scale=None, err_flag=None, stream=None):
    """Error-aware routing scores ln(err_ij / n_j) into ``t.scores`` (needs the pooled
    query centroids)."""
    scale = 1.0 / math.sqrt(p.d) if scale is None else scale
    C.sparse_attn_ear_scores(t.qbar, k, v, p.B, p.H, p.nqb, p.Nk, p.d, p.block, scale,
                             t.scores, err_flag, stream)


def route(p: Problem, t: Tables, kv_idx, kv_cnt, mode: str, rho=(1, 4), tau=0.9, scale=None,
          stream=None):
    scale = 1.0 / math.sqrt(p.d) if scale is None else scale
    if mode == "ear":
        C.sparse_attn_route_scores(t.scores, p.B, p.H, p.nqb, p.nkb, rho[0], rho[1], kv_idx,
                                   kv_cnt, kv_idx.shape[-1], stream)
        return
    if mode == "topk_cov":
        C.sparse_attn_route_cov(t.qbar, t.kbar_t, t.cov, p.B, p.H, p.nqb, p.nkb, p.d, rho[0],
                                rho[1], scale, kv_idx, kv_cnt, kv_idx.shape[-1], stream)
        return
    m = C.SA_ROUTE_TOPK if mode == "topk" else C.SA_ROUTE_MASS
    C.sparse_attn_route(t.qbar, t.kbar_t, p.B, p.H, p.nqb, p.nkb, p.d, m, rho[0], rho[1], tau,
                        scale, kv_idx, kv_cnt, kv_idx.shape[-1], stream)


def structured_mask(p: Problem, kv_idx, kv_cnt, frame_tokens, n_frames, window, n_anchors, period,
                    step, q_frame0=0, budget=0, stream=None):
    """Window + rotating anchors; budget > 0 uses the adaptive (extended) windows."""
    if budget:
        C.sparse_attn_structured_mask_adaptive(p.B, p.H, p.Nq, p.Nk, p.block, frame_tokens,
                                               n_frames, window, n_anchors, period, step, q_frame0,
                                               budget, kv_idx, kv_cnt, kv_idx.shape[-1], stream)
        return
    C.sparse_attn_structured_mask(p.B, p.H, p.Nq, p.Nk, p.block, frame_tokens, n_frames, window,
                                  n_anchors, period, step, q_frame0, kv_idx, kv_cnt,
                                  kv_idx.shape[-1], stream)


def forward(q, k, v, p: Problem, t: Tables, kv_idx, kv_cnt, out, scale=None, err_flag=None,
            stream=None, splits: int = 1, work=None):
    """The forward; ``splits`` > 1 shares every query tile's key blocks among that many
    CTAs and merges their partial results (``work``: fp32 scratch of at least
    ``sparse_attn_forward_work_bytes`` bytes)."""
    scale = 1.0 / math.sqrt(p.d) if scale is None else scale
    dt = C.SA_OUT_F32 if out.dtype == torch.float32 else C.SA_OUT_BF16
    m = t.hbar16 if p.order == 2 else t.M
    if splits > 1:
        C.sparse_attn_forward_split(q, k, t.v16, t.kbar16, t.vsum16, m, kv_idx, kv_cnt,
                                    kv_idx.shape[-1], p.B, p.H, p.Nq, p.Nk, p.d, p.block, p.order,
                                    scale, splits, work, out, dt, err_flag, stream)
    else:
        C.sparse_attn_forward(q, k, t.v16, t.kbar16, t.vsum16, m, kv_idx, kv_cnt, kv_idx.shape[-1],
                              p.B, p.H, p.Nq, p.Nk, p.d, p.block, p.order, scale, out, dt, err_flag,
                              stream)


@functools.lru_cache(maxsize=256)
def _plan(B, H, Nq, Nk, d, block, sms):
    return C.sparse_attn_forward_split_plan(B, H, Nq, Nk, d, block, sms)


def split_plan(p: Problem, device) -> tuple:
    """(splits, work bytes) the library picks for this shape on ``device``'s SMs."""
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    return _plan(p.B, p.H, p.Nq, p.Nk, p.d, p.block, sms)


class BlockSparseAttention:
    """Reusable buffers plus the three-stage call for one problem shape.

    mode "topk" keeps ceil(rho * nkb) blocks per query block, "topk_cov" the same
    number by the covariance-aware score (order 2), "ear" the same number by the
    error of the centroid approximation per token (SVG-EAR), "mass" the shortest
    prefix covering tau of the pooled softmax, "structured" the window + rotating
    anchor geometry given in ``geometry`` (frame_tokens, n_frames, window, budget,
    n_anchors, period, q_frame0) at the step passed to :meth:`__call__`.
    ``clusters`` = (C_q, C_k, iters) first clusters Q and K by k-means and runs the
    three stages on their group-major copies (V follows K), returning the output in the
    original query order. ``splits`` = key-range splits of the forward: None lets the
    library choose per call shape (:func:`split_plan`), an int fixes it.
    """

    def __init__(self, p: Problem, mode: str, rho=(1, 4), tau=0.9, geometry=None,
                 out_dtype=torch.float32, device="cuda", clusters=None, splits=None):
        self.p, self.mode, self.rho, self.tau, self.geometry = p, mode, rho, tau, geometry
        self.clusters = clusters
        self.splits, self._work, self.last_splits = splits, None, 1
        if mode == "topk_cov" and p.order != 2:
            raise ValueError("covariance-aware routing needs order 2 (the covariance norms)")
        if mode in ("topk", "topk_cov", "ear"):
            cap = -(-rho[0] * p.nkb // rho[1])
        else:
            cap = p.nkb
        self.tables = allocate_tables(p, device, ear=mode == "ear")
        self.kv_idx, self.kv_cnt = allocate_lists(p, cap, device)
        self.out = torch.empty(p.B, p.H, p.Nq, p.d, dtype=out_dtype, device=device)
        self.err_flag = torch.zeros(1, dtype=torch.int32, device=device)
        if clusters:
            # cluster-permuted layout: (C_q, C_k, iters); blocks are cut from the
            # group-major order of each tensor's k-means labels
            if mode == "structured":
                raise ValueError("the structured mask works on frame order, not on clusters")
            cq, ck, iters = clusters
            self.cl_q = allocate_clustering(p.B, p.H, p.Nq, p.d, cq, iters, device)
            self.cl_k = allocate_clustering(p.B, p.H, p.Nk, p.d, ck, iters, device)
            bf = dict(dtype=torch.bfloat16, device=device)
            self.q_p = torch.empty(p.B, p.H, p.Nq, p.d, **bf)
            self.k_p = torch.empty(p.B, p.H, p.Nk, p.d, **bf)
            self.v_p = torch.empty(p.B, p.H, p.Nk, p.d, **bf)
            self.out_p = torch.empty_like(self.out)

    def cluster(self, q, k, v, stream=None):
        """k-means of Q and K and the group-major copies of Q, K and V (every head)."""
        kmeans(q, self.cl_q, self.err_flag, stream)
        kmeans(k, self.cl_k, self.err_flag, stream)
        permute_rows(q, self.cl_q.perm, self.q_p, True, stream)
        permute_rows(k, self.cl_k.perm, self.k_p, True, stream)
        permute_rows(v, self.cl_k.perm, self.v_p, True, stream)
        return self.q_p, self.k_p, self.v_p

    def __call__(self, q, k, v, step: int = 0, stream=None) -> torch.Tensor:
        _check_inputs(q, k, v)
        self._run(q, k, v, self.out, None, step, stream)
        return self.out

    def _run(self, q, k, v, out, heads, step, stream):
        """All stages for the heads ``heads`` = (b, h0, h1) (None: every head). A head
        range runs as a problem of its own on views of every buffer; heads never
        interact, so any split of them gives the same output."""
        if heads is None:
            p, t, idx, cnt = self.p, self.tables, self.kv_idx, self.kv_cnt
            sub = lambda x: x
        else:
            b, h0, h1 = heads
            p = dataclasses.replace(self.p, B=1, H=h1 - h0)
            sub = lambda x: None if x is None else x[b:b + 1, h0:h1]
            t = Tables(**{f.name: sub(getattr(self.tables, f.name))
                          for f in dataclasses.fields(Tables)})
            idx, cnt = sub(self.kv_idx), sub(self.kv_cnt)
            q, k, v, out = sub(q), sub(k), sub(v), sub(out)
        if self.clusters:
            clq = dataclasses.replace(self.cl_q, centroids=sub(self.cl_q.centroids),
                                      labels=sub(self.cl_q.labels), perm=sub(self.cl_q.perm),
                                      offsets=sub(self.cl_q.offsets))
            clk = dataclasses.replace(self.cl_k, centroids=sub(self.cl_k.centroids),
                                      labels=sub(self.cl_k.labels), perm=sub(self.cl_k.perm),
                                      offsets=sub(self.cl_k.offsets))
            qp, kp, vp, op_ = sub(self.q_p), sub(self.k_p), sub(self.v_p), sub(self.out_p)
            kmeans(q, clq, self.err_flag, stream)
            kmeans(k, clk, self.err_flag, stream)
            permute_rows(q, clq.perm, qp, True, stream)
            permute_rows(k, clk.perm, kp, True, stream)
            permute_rows(v, clk.perm, vp, True, stream)
            self._attend(p, t, idx, cnt, qp, kp, vp, op_, step, stream)
            permute_rows(op_, clq.perm, out, False, stream)
        else:
            self._attend(p, t, idx, cnt, q, k, v, out, step, stream)

    def _attend(self, p, t, kv_idx, kv_cnt, q, k, v, out, step, stream):
        pool(q if self.mode != "structured" else None, k, v, p, t, stream,
             err_flag=self.err_flag)
        if self.mode == "structured":
            g = self.geometry
            structured_mask(p, kv_idx, kv_cnt, g["frame_tokens"], g["n_frames"],
                            g["window"], g["n_anchors"], g["period"], step, g.get("q_frame0", 0),
                            g.get("budget", 0), stream)
        else:
            if self.mode == "ear":
                ear_scores(k, v, p, t, err_flag=self.err_flag, stream=stream)
            route(p, t, kv_idx, kv_cnt, self.mode, self.rho, self.tau, stream=stream)
        self.forward_stage(p, t, kv_idx, kv_cnt, q, k, v, out, stream)

    def forward_stage(self, p, t, kv_idx, kv_cnt, q, k, v, out, stream=None):
        """The forward of one (sub-)problem, split as :attr:`splits` says. The automatic
        choice is made for the whole problem, also when a head range runs on its own, so
        that every form of the call computes each row the same way (bit for bit). The
        scratch for the partial results is kept and only grows."""
        S = self.splits if self.splits is not None else split_plan(self.p, self.out.device)[0]
        work = None
        if S > 1:
            need = C.sparse_attn_forward_work_bytes(p.B, p.H, p.Nq, p.d, S) // 4
            if self._work is None or self._work.numel() < need:
                self._work = torch.empty(need, dtype=torch.float32, device=self.out.device)
            work = self._work
            if isinstance(stream, torch.cuda.Stream):
                work.record_stream(stream)
        self.last_splits = S
        forward(q, k, v, p, t, kv_idx, kv_cnt, out, err_flag=self.err_flag, stream=stream,
                splits=S, work=work)

    def capture(self, q, k, v, step: int = 0) -> "torch.cuda.CUDAGraph":
        """Record one call on these buffers as a CUDA graph: replaying it repeats every
        launch of the call (for the step given) on whatever the buffers hold then, with no
        host work per launch."""
        dev = self.out.device
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):   # one eager call first: attributes, tensor maps
            self(q, k, v, step=step)
        torch.cuda.current_stream(dev).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self(q, k, v, step=step)
        return g

    def run_from_host(self, q_h, k_h, v_h, out_h, step: int = 0, chunks: int = 10):
        """One call with Q, K, V in (pinned) host memory and the output written to the
        (pinned) host tensor ``out_h``.

        The heads are split into ranges of four (``chunks`` ranges or fewer): the
        host-to-device copies run ahead on one stream, each range is computed on the
        current stream as soon as its inputs are in, and its output goes back on a third
        stream while the next range computes. Successive calls alternate between two
        sets of device input and output buffers, so the next call's inputs load while
        this call computes and its outputs drain while the next one computes. Returns
        after enqueueing; call :meth:`wait_host_copies` (or synchronise) before reading
        ``out_h``."""
        p = self.p
        dev = self.out.device
        if getattr(self, "_sets", None) is None:
            mk = lambda x: torch.empty(x.shape, dtype=x.dtype, device=dev)
            self._sets = [dict(q=mk(q_h), k=mk(k_h), v=mk(v_h), out=torch.empty_like(self.out),
                               free_in=None, free_out=None) for _ in range(2)]
            self._h2d, self._d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            self._call = 0
        st = self._sets[self._call % 2]
        self._call += 1
        q, k, v, out = st["q"], st["k"], st["v"], st["out"]
        cs = torch.cuda.current_stream(dev)
        # Head ranges start at multiples of 4 heads of the flattened (batch, head) index,
        # so that every per-head table slice starts on a 16-byte boundary (the C ABI's
        # alignment rule); otherwise the call runs as one range.
        per_b = max(1, -(-chunks // p.B))              # ranges per batch entry
        step_h = -(-(-(-p.H // per_b)) // 4) * 4
        ranges = [(b, h0, min(p.H, h0 + step_h)) for b in range(p.B)
                  for h0 in range(0, p.H, step_h)]
        if any((b * p.H + h0) % 4 for b, h0, _ in ranges):
            ranges = [(b, 0, p.H) for b in range(p.B)] if (p.H % 4 == 0) else [None]
        # this set's inputs may still be read by the compute of the call before last, and
        # its output may still be draining to the host
        if st["free_in"] is not None:
            self._h2d.wait_event(st["free_in"])
        if st["free_out"] is not None:
            cs.wait_event(st["free_out"])
        ready = []
        with torch.cuda.stream(self._h2d):
            for r in ranges:
                sl = (slice(None),) if r is None else (r[0], slice(r[1], r[2]))
                for dst, src in ((q, q_h), (k, k_h), (v, v_h)):
                    dst[sl].copy_(src[sl], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self._h2d)
                ready.append(ev)
        for r, ev in zip(ranges, ready):
            cs.wait_event(ev)
            self._run(q, k, v, out, r, step, None)
            done = torch.cuda.Event()
            done.record(cs)
            self._d2h.wait_event(done)
            with torch.cuda.stream(self._d2h):
                sl = (slice(None),) if r is None else (r[0], slice(r[1], r[2]))
                out_h[sl].copy_(out[sl], non_blocking=True)
        st["free_in"] = torch.cuda.Event()
        st["free_in"].record(cs)
        st["free_out"] = torch.cuda.Event()
        st["free_out"].record(self._d2h)
        return out_h

    def wait_host_copies(self):
        """Make the current stream wait for every output copy to the host issued so far."""
        if getattr(self, "_d2h", None) is not None:
            torch.cuda.current_stream(self.out.device).wait_stream(self._d2h)

    def check(self):
        """Raise if an earlier call failed on the device (synchronises): SA_ERR_RANGE when a
        pooled fp16 table value did not fit (the output is then not valid), SA_ERR_TIMEOUT
        when a bounded device wait gave up. The flag is sticky: it stays set until cleared
        with ``err_flag.zero_()``."""
        flag = int(self.err_flag.item())
        if flag & C.SA_FLAG_RANGE:
            raise C.SparseAttnError(C.SA_ERR_RANGE, "a pooled fp16 table value (V copy, value "
                                    "sum or M_j) does not fit in fp16 (|x| >= 65520); scale V "
                                    f"down by a power of two (flag {flag:#x})")
        if flag:
            raise C.SparseAttnError(C.SA_ERR_TIMEOUT, f"device wait timed out (flag {flag:#x})")
