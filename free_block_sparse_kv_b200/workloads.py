"""Seeded synthetic workloads for block-sparse attention with skipped-block compensation.

This module only draws random inputs. It holds none of the method's arithmetic
(no pooling, no routing, no attention), so both the fp64 oracle checks and the
GPU path can take their inputs from it.

Every tensor is drawn per (batch, head) from its own counter-keyed PCG64 stream,
``SeedSequence([seed, tensor_id, b, h])``. One head can therefore be regenerated
on the host without drawing the whole workload, which is how the full-size
parity tests sample heads.

Token order is frame-major, then row, then column, as in a video DiT latent.
Values are drawn in fp32 and rounded to bf16 (round to nearest even). The
rounded values are returned as fp32 arrays (exactly representable) together
with their bf16 bit patterns.

The five workloads follow the attention calls that the pages measure on
(video DiTs and an autoregressive world model; PISA §4, LVSA §4, SVG-EAR §4):
their trained models and video suites are not available, so clustered Gaussian
tokens of the same shapes stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Counter keys for the per-head streams. Adding a tensor means a new key, so the
# existing streams never change.
_Q, _K, _V = 1, 2, 3


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention call: shapes, blocking, keep rule and value recipe."""

    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    block: int
    order: int                      # 0 or 1: compensation order for skipped blocks
    mode: str                       # "topk", "topk_cov", "ear", "mass" or "structured"
    rho: tuple = (1, 4)             # keep fraction rho_num / rho_den (topk)
    tau: float = 0.9                # covered mass (mass)
    recipe: str = "blocks"          # "blocks", "patches" or "drift"
    grid: Optional[tuple] = None    # (frames, rows, cols) of the KV token grid
    patch: tuple = (4, 4, 4)        # patch extent (frames, rows, cols) for "patches"
    noise: float = 0.3
    outlier_p: float = 0.0          # fraction of key rows scaled by outlier_scale
    outlier_scale: float = 4.0
    drift: float = 0.05             # per-frame center random walk ("drift")
    q_frame0: int = 0               # first frame of the query chunk
    # structured (LVSA-style) mask geometry
    window: int = 3
    n_anchors: int = 4
    period: int = 10
    budget: int = 0                 # > 0: adaptive windows reaching |A(t)| = budget frames
    clusters: tuple = ()            # (C_q, C_k, iters): k-means group-major layout first
    steps: tuple = (0,)
    seed: int = 0

    @property
    def nqb(self) -> int:
        return -(-self.Nq // self.block)

    @property
    def nkb(self) -> int:
        return -(-self.Nk // self.block)

    @property
    def frame_tokens(self) -> int:
        return self.grid[1] * self.grid[2] if self.grid else 0

    @property
    def n_frames(self) -> int:
        return self.grid[0] if self.grid else 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def keep(self) -> int:
        """Blocks kept per query block under top-rho: ceil(rho * nkb) in integers."""
        num, den = self.rho
        return -(-num * self.nkb // den)

    def cap(self) -> int:
        """Row capacity of the kept-index lists."""
        return self.keep() if self.mode in ("topk", "topk_cov", "ear") else self.nkb

    def dense_flops(self) -> float:
        """Dense-equivalent attention flops of one call: 4 * B * H * Nq * Nk * d."""
        return 4.0 * self.B * self.H * self.Nq * self.Nk * self.d


WORKLOADS = {
    # Small case: per-64-token-block key/query centers.
    "uniform-4k": Workload(
        name="uniform-4k", B=1, H=2, Nq=4096, Nk=4096, d=64, block=64, order=0,
        mode="topk", rho=(1, 4), recipe="blocks"),
    # Video-DiT self-attention on a 21x30x52 latent grid.
    "dit-21x30x52": Workload(
        name="dit-21x30x52", B=1, H=24, Nq=32760, Nk=32760, d=128, block=128, order=1,
        mode="topk", rho=(1, 5), recipe="patches", grid=(21, 30, 52)),
    # 720p-scale video-DiT attention on a 21x45x80 grid with 5% outlier keys.
    "dit720p-21x45x80": Workload(
        name="dit720p-21x45x80", B=1, H=40, Nq=75600, Nk=75600, d=128, block=128, order=1,
        mode="topk", rho=(1, 10), recipe="patches", grid=(21, 45, 80), outlier_p=0.05),
    # The same 720p call with PISA's hybrid order: the global first-order matrix for every
    # skipped block and covariance-aware top-k.
    "dit720p-hybrid-21x45x80": Workload(
        name="dit720p-hybrid-21x45x80", B=1, H=40, Nq=75600, Nk=75600, d=128, block=128, order=2,
        mode="topk_cov", rho=(1, 10), recipe="patches", grid=(21, 45, 80), outlier_p=0.05),
    # The same 720p call with SVG-EAR's routing: blocks ranked by the error of their
    # centroid approximation per token, order-0 (centroid) compensation for the rest.
    "dit720p-ear-21x45x80": Workload(
        name="dit720p-ear-21x45x80", B=1, H=40, Nq=75600, Nk=75600, d=128, block=128, order=0,
        mode="ear", rho=(1, 10), recipe="patches", grid=(21, 45, 80), outlier_p=0.05),
    # The 720p call on the cluster-permuted layout: Q and K grouped by k-means into 296
    # clusters each (about two blocks per cluster), three Lloyd updates, then blocks cut
    # from the group-major order.
    "dit720p-kmeans-21x45x80": Workload(
        name="dit720p-kmeans-21x45x80", B=1, H=40, Nq=75600, Nk=75600, d=128, block=128,
        order=1, mode="topk", rho=(1, 10), recipe="patches", grid=(21, 45, 80), outlier_p=0.05,
        clusters=(296, 296, 3)),
    # Long video with a local window and rotating anchor frames (denoising steps 0..9).
    "longvideo-41x30x52": Workload(
        name="longvideo-41x30x52", B=1, H=12, Nq=63960, Nk=63960, d=128, block=128, order=0,
        mode="structured", recipe="patches", grid=(41, 30, 52), window=3, n_anchors=4,
        period=10, steps=tuple(range(10))),
    # The same long video with LVSA's extended adaptive windows: every frame attends to
    # 11 frames (4 anchors + 7 window frames), windows growing past anchors and edges.
    "longvideo-adaptive-41x30x52": Workload(
        name="longvideo-adaptive-41x30x52", B=1, H=12, Nq=63960, Nk=63960, d=128, block=128,
        order=0, mode="structured", recipe="patches", grid=(41, 30, 52), window=3, n_anchors=4,
        period=10, budget=11, steps=tuple(range(10))),
    # Autoregressive world-model chunk: frame 40 attends to frames 0..40.
    "worldmodel-chunk": Workload(
        name="worldmodel-chunk", B=4, H=16, Nq=1560, Nk=63960, d=128, block=64, order=1,
        mode="mass", tau=0.9, recipe="drift", grid=(41, 30, 52), patch=(1, 4, 4), q_frame0=40),
}

# The workload the throughput metric is quoted on.
METRIC_WORKLOAD = "dit720p-21x45x80"


def bf16_round(x: np.ndarray):
    """Round fp32 to bf16 (nearest, ties to even). Returns (values as fp32, uint16 bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bits = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return vals, bits


def _rng(w: Workload, tensor: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, tensor, b, h])))


def _patch_ids(w: Workload, first_token: int, n_tokens: int) -> tuple:
    """Patch id of each token of a frame-major grid, and the number of patches."""
    F, R, C = w.grid
    pf, pr, pc = w.patch
    t = np.arange(first_token, first_token + n_tokens)
    f, rem = np.divmod(t, R * C)
    y, x = np.divmod(rem, C)
    nr, nc = -(-R // pr), -(-C // pc)
    nf = -(-F // pf)
    return (f // pf) * (nr * nc) + (y // pr) * nc + (x // pc), nf * nr * nc


def _clustered(w: Workload, rng: np.random.Generator, first_token: int, n_tokens: int) -> np.ndarray:
    """Queries or keys: a center per cluster plus noise * N(0, 1). Centers are drawn first."""
    d = w.d
    if w.recipe == "blocks":
        n_blk = -(-n_tokens // w.block)
        centers = rng.standard_normal((n_blk, d), dtype=np.float32)
        ids = np.arange(n_tokens) // w.block
        noise = rng.standard_normal((n_tokens, d), dtype=np.float32)
        return centers[ids] + np.float32(w.noise) * noise
    if w.recipe == "patches":
        ids, n_patch = _patch_ids(w, first_token, n_tokens)
        centers = rng.standard_normal((n_patch, d), dtype=np.float32)
        noise = rng.standard_normal((n_tokens, d), dtype=np.float32)
        return centers[ids] + np.float32(w.noise) * noise
    if w.recipe == "drift":
        # Spatial patches per frame; each patch center takes a random walk over frames:
        # c[p, 0] ~ N(0, I), c[p, f] = c[p, f-1] + drift * N(0, I).
        F, R, C = w.grid
        _, pr, pc = w.patch
        n_sp = (-(-R // pr)) * (-(-C // pc))
        walk = rng.standard_normal((F, n_sp, d), dtype=np.float32)
        walk[1:] *= np.float32(w.drift)
        centers = np.cumsum(walk, axis=0, dtype=np.float32)
        t = np.arange(first_token, first_token + n_tokens)
        f, rem = np.divmod(t, R * C)
        y, x = np.divmod(rem, C)
        sp = (y // pr) * (-(-C // pc)) + (x // pc)
        noise = rng.standard_normal((n_tokens, d), dtype=np.float32)
        return centers[f, sp] + np.float32(w.noise) * noise
    raise ValueError(f"unknown recipe {w.recipe!r}")


def _head_f32(w: Workload, b: int, h: int):
    """Unrounded fp32 draws of one head (see :func:`head_inputs` for the order)."""
    q_first = w.q_frame0 * w.frame_tokens
    q = _clustered(w, _rng(w, _Q, b, h), q_first, w.Nq)
    rk = _rng(w, _K, b, h)
    k = _clustered(w, rk, 0, w.Nk)
    if w.outlier_p > 0.0:
        rows = rk.random(w.Nk) < w.outlier_p
        k[rows] *= np.float32(w.outlier_scale)
    v = _rng(w, _V, b, h).standard_normal((w.Nk, w.d), dtype=np.float32)
    return q, k, v


def head_inputs_bits(w: Workload, b: int, h: int):
    """bf16 bit patterns (uint16) of Q [Nq, d], K [Nk, d], V [Nk, d] of one head."""
    return tuple(bf16_round(x)[1] for x in _head_f32(w, b, h))


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact fp32 values of bf16 bit patterns."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def head_inputs(w: Workload, b: int, h: int):
    """Q [Nq, d], K [Nk, d], V [Nk, d] of one (batch, head), bf16-rounded, as fp32 arrays.

    Draw order within the head: Q centers, Q noise, K centers, K noise, outlier
    mask, V. Q and K draw independent centers from the same distribution.
    """
    return tuple(bits_to_f32(x) for x in head_inputs_bits(w, b, h))


def full_inputs_bits(w: Workload, heads=None, threads: int = 0):
    """bf16 bits of Q [B,H,Nq,d], K and V [B,H,Nk,d] for the whole workload.

    ``heads`` optionally limits the draw to a list of (b, h) pairs; the other heads
    are left zero. Heads are drawn on ``threads`` threads (default: the usable
    cores); each head's stream is independent, so the result does not depend on it.
    """
    import concurrent.futures
    import os
    q = np.zeros((w.B, w.H, w.Nq, w.d), dtype=np.uint16)
    k = np.zeros((w.B, w.H, w.Nk, w.d), dtype=np.uint16)
    v = np.zeros((w.B, w.H, w.Nk, w.d), dtype=np.uint16)
    todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]

    def one(bh):
        b, h = bh
        q[b, h], k[b, h], v[b, h] = head_inputs_bits(w, b, h)

    n = threads or max(1, min(32, len(os.sched_getaffinity(0))))
    with concurrent.futures.ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(one, todo))
    return q, k, v


def shrink(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **changes)
