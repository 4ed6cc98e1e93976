"""Benchmark: one step = pool -> route (or structured mask) -> forward over one
synthetic workload, on each GPU (weak scaling: every rank runs its own copy of
the workload, seeded by its rank; no collective on the data path).

Prints one JSON line on rank 0. `value` is dense-equivalent attention TFLOPS
(4 * B * H * Nq * Nk * d per call) summed over ranks, timed with CUDA events
on the launching stream (max over ranks), inputs resident in HBM. `e2e` is the
same metric through the public API with pinned host buffers, including the
host-to-device copy of Q, K, V and the device-to-host copy of the output.

--impl reference times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_block_sparse_kv_b200 import workloads as W  # noqa: E402

METRIC = "dense-equiv attention TFLOPS & ms/call at N=75,600 d=128; % of bf16 TC peak"
UNIT = "TFLOPS"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.METRIC_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--graphs", action="store_true",
                    help="also time the step replayed from CUDA graphs (reported as 'graph')")
    ap.add_argument("--splits", type=int, default=0,
                    help="key-range splits of the forward (0: the library's choice)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run on this many heads instead of the workload's (profiler captures)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure only --workload (by default the metric workload's line also "
                         "carries the other configurations under 'workloads')")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(bf16=d["bf16_tflops"], bf16_sustained=d["bf16_tflops_sustained"],
                    hbm=d["hbm_gbs"], source="measured")
    return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# ---------------------------------------------------------------------------
# work model
# ---------------------------------------------------------------------------

def executed_flops(w: W.Workload, kv_idx: np.ndarray, kv_cnt: np.ndarray) -> dict:
    """MMA flops the forward executes for the given kept lists (per launch).

    exact kept block j, query block i:     4 * nq_i * n_j * d
    skipped block, order 0 (logit + value): 4 * nq_i * d
    skipped block, order 1 (q M_j):         2 * nq_i * d * d
    order 2 (q Hbar, once per query block with a skipped block): 2 * nq_i * d * d
    """
    nq = np.array([min(w.block, w.Nq - i * w.block) for i in range(w.nqb)], np.float64)
    nk = np.array([min(w.block, w.Nk - j * w.block) for j in range(w.nkb)], np.float64)
    exact = order0 = order1 = 0.0
    for b in range(kv_cnt.shape[0]):
        for h in range(kv_cnt.shape[1]):
            for i in range(w.nqb):
                c = int(kv_cnt[b, h, i])
                kept = kv_idx[b, h, i, :c]
                tok = nk[kept].sum()
                exact += 4.0 * nq[i] * tok * w.d
                skipped = w.nkb - c
                order0 += 4.0 * nq[i] * w.d * skipped
                if w.order == 1:
                    order1 += 2.0 * nq[i] * w.d * w.d * skipped
                elif w.order == 2 and skipped:
                    order1 += 2.0 * nq[i] * w.d * w.d
    return dict(exact=exact, order0=order0, order1=order1, total=exact + order0 + order1)


FORWARD_SOURCES = ("forward_tc.cu", "tc.cuh", "common.cuh", "tmap.h")


def forward_sources_sha256() -> str:
    """Hash of the forward kernel's sources, to tell whether a DRAM capture still applies."""
    h = hashlib.sha256()
    for name in FORWARD_SOURCES:
        with open(os.path.join(ROOT, "free_block_sparse_kv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def forward_traffic(w: W.Workload):
    """DRAM bytes (read + write) of one forward launch on this workload, from the ncu capture
    summarised under profiles/, or None when there is none or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", f"forward_dram_{w.name}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, _, val = line.strip().partition(":")
                vals[key.strip("- `")] = val.strip().strip("`")
    try:
        if vals.get("sources_sha256") != forward_sources_sha256():
            return None
        return float(vals["dram_bytes_read_per_launch"]) + float(vals["dram_bytes_write_per_launch"])
    except (KeyError, ValueError):
        return None


def pool_bytes(w: W.Workload, with_q: bool) -> float:
    """Algorithmic HBM bytes of one pool stage, as the method defines its tables: read K, V
    (and Q); write the query centroids, the KV centroids and value sums in fp32 with one
    16-bit copy of each for the tensor cores, and (order 1 or 2) the first-order matrices
    M_j in 16 bits; for order 2 also the two passes over M (global matrix, covariance
    norms). Bytes this library writes beyond that are in :func:`pool_extra_bytes`."""
    bh = w.B * w.H
    rd = bh * w.Nk * w.d * 2 * 2 + (bh * w.Nq * w.d * 2 if with_q else 0)
    wr = bh * w.nkb * w.d * (4 + 4 + 2 + 2) + (bh * w.nqb * w.d * 4 if with_q else 0)
    if w.order >= 1:
        wr += bh * w.nkb * w.d * w.d * 2
    if w.order == 2:  # the global matrix and the covariance norms read the M table twice
        rd += 2 * bh * w.nkb * w.d * w.d * 2
        wr += bh * w.d * w.d * 6 + bh * w.nkb * 4
    return float(rd + wr)


def pool_extra_bytes(w: W.Workload) -> dict:
    """Bytes the pool writes beyond the method's tables: the fp16 copy of V (the operand
    of the forward's exact value products) and the second (low) bf16 plane of the
    centroids."""
    bh = w.B * w.H
    return {"v16": float(bh * w.Nk * w.d * 2), "kbar16_lo": float(bh * w.nkb * w.d * 2)}


def route_work(w: W.Workload):
    """Algorithmic bytes (read the centroid tables, write the lists) and fp32 flops of one
    route stage (scoring GEMM 2 nqb nkb d per head)."""
    bh = w.B * w.H
    by = bh * (w.nqb + w.nkb) * w.d * 4 + bh * w.nqb * (w.cap() + 1) * 4
    if w.mode == "ear":   # reads the score table instead of the centroid tables
        by = bh * w.nqb * w.nkb * 4 + bh * w.nqb * (w.cap() + 1) * 4
    fl = 0.0 if w.mode in ("ear", "structured") else 2.0 * bh * w.nqb * w.nkb * w.d
    return float(by), fl


# fp32 FMA peak of the part from its unit counts and clock: 148 SMs x 128 fp32 lanes x 2
# flops x 1.965 GHz
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def kv_cached_start(w: W.Workload) -> int:
    """First KV block of a chunk appended to a frame cache (world model), else 0."""
    if not w.frame_tokens or not w.q_frame0 or w.Nk <= w.q_frame0 * w.frame_tokens:
        return 0
    return (w.q_frame0 * w.frame_tokens) // w.block


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------

class OracleSampler:
    """The fp64 oracle on one head of a workload: pooling and routing once, then query
    rows (spread over the head in a fixed random order) forwarded in samples."""

    def __init__(self, w: W.Workload):
        from oracle import block_sparse_attention as O
        self.O, self.w = O, w
        q, k, v = W.head_inputs(w, 0, 0)
        t0 = time.perf_counter()
        if w.clusters:
            from oracle import cluster_layout as K
            cq, ck, iters = w.clusters
            pq = K.group_major_permutation(K.kmeans(q, cq, iters)[0], cq)[0]
            pk = K.group_major_permutation(K.kmeans(k, ck, iters)[0], ck)[0]
            q, k, v = q[pq], k[pk], v[pk]
        if w.mode == "structured":
            self.kept = O.structured_kept(w.Nq, w.Nk, w.block, w.frame_tokens, w.n_frames,
                                          w.window, w.n_anchors, w.period, 0, w.q_frame0,
                                          budget=w.budget)
        else:
            self.kept = O.route_head(q, k, w.block, w.mode, w.scale, keep=w.keep(), tau=w.tau,
                                     v=v)[0]
        self.tables = O.pool_keys_values(k, v, w.block, min(w.order, 1))
        self.hbar = O.global_first_order(self.tables[3]) if w.order == 2 else None
        self.t_setup = time.perf_counter() - t0
        self.q64, self.k, self.v = q.astype(np.float64), k, v
        self.order = np.random.default_rng(0).permutation(w.Nq)
        self.done = 0

    def rows(self, n: int) -> int:
        """Forward the next n rows (wrapping around the head); returns n."""
        w = self.w
        kbar, vsum, counts, mats = self.tables
        left = n
        while left > 0:
            start = self.done % w.Nq
            take = min(left, 16, w.Nq - start)
            rows = self.order[start:start + take]
            self.O.forward_rows(self.q64[rows], rows // w.block, self.k, self.v, kbar, vsum,
                                counts, mats, self.kept, w.block, w.order, w.scale,
                                hbar=self.hbar)
            self.done += take
            left -= take
        return n

    def tflops(self, rows: int, seconds: float) -> float:
        """Dense-equivalent TFLOPS of `rows` rows forwarded in `seconds`, with the head's
        pooling and routing amortised over its Nq rows."""
        per_row = seconds / rows + self.t_setup / self.w.Nq
        return 4.0 * self.w.Nk * self.w.d / per_row / 1e12

    def ms_per_call(self, rows: int, seconds: float) -> float:
        """A whole call (every row of every head) extrapolated from the rate measured."""
        w = self.w
        return (seconds / rows + self.t_setup / w.Nq) * w.Nq * w.B * w.H * 1e3


def host_info() -> dict:
    try:
        blas = ",".join(sorted({c.get("internal_api", "?") for c in
                                __import__("threadpoolctl").threadpool_info()}))
    except Exception:  # the report is informational
        blas = "unknown"
    return dict(cores=len(os.sched_getaffinity(0)), cpu_count=os.cpu_count(), blas=blas)


def time_oracle(w: W.Workload, seconds: float) -> dict:
    """Time the fp64 oracle on a bounded sample: one head's pooling and routing, then query
    rows until `seconds` have passed. Scaled to dense-equivalent TFLOPS: rows * Nk * d * 4
    per second of the oracle's time."""
    smp = OracleSampler(w)
    t1 = time.perf_counter()
    done = 0
    while done < w.Nq and time.perf_counter() - t1 < seconds:
        done += smp.rows(16)
    t_rows = time.perf_counter() - t1
    return dict(value=smp.tflops(done, t_rows), unit=UNIT, **host_info(), kind="oracle",
                sample=f"{w.name}: head (0,0) {'clustered, ' if w.clusters else ''}pooled and "
                       f"routed ({smp.t_setup:.1f} s), then {done} of "
                       f"{w.Nq} query rows forwarded ({t_rows:.1f} s); scaled per row to the "
                       f"dense-equivalent flops of one call",
                seconds=smp.t_setup + t_rows, ms_per_call_est=smp.ms_per_call(done, t_rows))


def reference_rows_per_step(seconds_per_row: float, budget_s: float, steps: int) -> int:
    """Rows per timed step so that `steps` steps take about `budget_s` seconds (at least 16,
    a whole number of 16-row chunks)."""
    rows = int(budget_s / max(steps, 1) / max(seconds_per_row, 1e-9))
    return max(16, rows - rows % 16)


def run_reference(args, w):
    """The reference arm: the fp64 oracle on the host cores. One step = one bounded sample
    of the workload (a fixed number of query rows of head (0,0)); W warm-up steps calibrate
    the sample size so that the K timed steps take about --cpu-seconds."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = OracleSampler(w)
    t0 = time.perf_counter()
    for _ in range(max(args.warmup, 1)):
        smp.rows(16)
    per_row = (time.perf_counter() - t0) / (16 * max(args.warmup, 1))
    rows_step = reference_rows_per_step(per_row, args.cpu_seconds, args.steps)
    step_s = []
    for _ in range(args.steps):
        t = time.perf_counter()
        smp.rows(rows_step)
        step_s.append(time.perf_counter() - t)
    total = float(sum(step_s))
    rows = rows_step * args.steps
    value = smp.tflops(rows, total)
    info = host_info()
    sample = (f"{w.name}: head (0,0) pooled and routed once ({smp.t_setup:.1f} s, amortised "
              f"over its {w.Nq} rows); each step forwards {rows_step} query rows of that head; "
              f"{args.steps} timed steps = {rows} rows in {total:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                   "block": w.block, "order": w.order, "mode": w.mode},
        "step": f"one bounded sample: {rows_step} query rows of head (0,0)",
        "rows_timed": rows,
        "ms_per_call_extrapolated": smp.ms_per_call(rows, total),
        "cpu_baseline": {"value": value, "unit": UNIT, **info, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

OTHER_CONFIGS = ("uniform-4k", "dit-21x30x52", "longvideo-41x30x52", "worldmodel-chunk")


def keep_label(w: W.Workload) -> str:
    if w.mode == "topk":
        return f"top {w.rho[0]}/{w.rho[1]}"
    if w.mode == "topk_cov":
        return f"top {w.rho[0]}/{w.rho[1]}, covariance-aware"
    if w.mode == "ear":
        return f"top {w.rho[0]}/{w.rho[1]}, error-aware"
    if w.mode == "mass":
        return f"mass {w.tau}"
    return "window+anchors" + (f", adaptive budget {w.budget}" if w.budget else "")


def launches_per_step(w: W.Workload, splits: int) -> int:
    """Kernels of one step: pool, route or mask, forward (+ the split merge); hybrid order
    adds the two passes over M, error-aware routing its probe, clustering 2 x (7 + 8 iters)
    k-means launches plus three gathers and the output scatter."""
    n = 5 if w.order == 2 else 4 if w.mode == "ear" else 3
    n += 1 if splits > 1 else 0
    if w.clusters:
        n += 2 * (7 + 8 * w.clusters[2]) + 4
    return n


class Session:
    """One GPU rank: device, stream and the collective helpers of dist.py."""

    def __init__(self):
        import torch
        from free_block_sparse_kv_b200 import dist as D
        self.torch, self.D = torch, D
        self.world, self.rank, local = D.env_ranks()
        torch.cuda.set_device(local)
        self.dev = torch.device("cuda", local)
        D.init("nccl", device=self.dev)
        self.stream = torch.cuda.current_stream(self.dev)
        props = torch.cuda.get_device_properties(self.dev)
        dev_id = str(getattr(props, "uuid", local))
        if dev_id and not dev_id.startswith("GPU-") and len(dev_id) == 36:
            dev_id = "GPU-" + dev_id
        self.dev_id = dev_id

    def barrier(self):
        self.D.barrier()

    def max(self, x: float) -> float:
        return self.D.max_over_ranks(x, device=self.dev)


class Bench:
    """A workload set up on one rank: pinned host inputs, device inputs, the operator."""

    def __init__(self, ses: Session, w: W.Workload, splits=None):
        torch = ses.torch
        from free_block_sparse_kv_b200 import attention as A
        self.A, self.ses, self.w = A, ses, w
        wr = ses.D.rank_workload(w, ses.rank)   # weak scaling: each rank its own problem
        qb, kb, vb = W.full_inputs_bits(wr)
        as_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        self.q_h, self.k_h, self.v_h = (as_t(x).pin_memory() for x in (qb, kb, vb))
        del qb, kb, vb
        self.q, self.k, self.v = (x.to(ses.dev) for x in (self.q_h, self.k_h, self.v_h))
        self.p = A.Problem(w.B, w.H, w.Nq, w.Nk, w.d, w.block, w.order)
        geometry = dict(frame_tokens=w.frame_tokens, n_frames=w.n_frames, window=w.window,
                        n_anchors=w.n_anchors, period=w.period, q_frame0=w.q_frame0,
                        budget=w.budget)
        self.op = A.BlockSparseAttention(self.p, w.mode, rho=w.rho, tau=w.tau,
                                         geometry=geometry if w.mode == "structured" else None,
                                         out_dtype=torch.float32, device=ses.dev,
                                         clusters=w.clusters or None, splits=splits)
        self.cycle = w.steps if w.mode == "structured" else (0,)

    def stage_step(self, s, ev):
        """One step with events around each stage: (clustering), pool, mask/route,
        forward, (output back to the query order)."""
        A, w, op, p, st = self.A, self.w, self.op, self.p, self.ses.stream
        use_q = w.mode != "structured"
        ev[0].record(st)
        qq, kk, vv, out = self.q, self.k, self.v, op.out
        if w.clusters:
            qq, kk, vv = op.cluster(self.q, self.k, self.v)
            out = op.out_p
        ev[5].record(st)
        A.pool(qq if use_q else None, kk, vv, p, op.tables)
        ev[1].record(st)
        if w.mode == "structured":
            A.structured_mask(p, op.kv_idx, op.kv_cnt, w.frame_tokens, w.n_frames, w.window,
                              w.n_anchors, w.period, s, w.q_frame0, budget=w.budget)
            ev[4].record(st)
        else:
            if w.mode == "ear":
                A.ear_scores(kk, vv, p, op.tables, err_flag=op.err_flag)
            ev[4].record(st)
            A.route(p, op.tables, op.kv_idx, op.kv_cnt, w.mode, w.rho, w.tau)
        ev[2].record(st)
        op.forward_stage(p, op.tables, op.kv_idx, op.kv_cnt, qq, kk, vv, out)
        ev[3].record(st)
        if w.clusters:
            A.permute_rows(op.out_p, op.cl_q.perm, op.out, gather=False)
        ev[6].record(st)

    def run(self, steps: int, warmup: int) -> dict:
        """W untimed steps, then `steps` timed steps between barriers (max over ranks)."""
        torch, ses = self.ses.torch, self.ses
        for i in range(warmup):
            self.op(self.q, self.k, self.v, step=self.cycle[i % len(self.cycle)])
        torch.cuda.synchronize(ses.dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ses.barrier()
        torch.cuda.synchronize(ses.dev)
        with ClockSampler(ses.dev_id) as clocks:
            start.record(ses.stream)
            for i in range(steps):
                self.stage_step(self.cycle[i % len(self.cycle)], evs[i])
            end.record(ses.stream)
            torch.cuda.synchronize(ses.dev)
        ses.barrier()
        self.op.check()
        mean = lambda a, b: float(np.mean([e[a].elapsed_time(e[b]) for e in evs]))
        per_call = [e[0].elapsed_time(e[6]) for e in evs]
        r = dict(ms_step=ses.max(start.elapsed_time(end) / steps), per_call=per_call,
                 pool=mean(5, 1), route=mean(1, 2), forward=mean(2, 3),
                 probe=mean(1, 4) if self.w.mode == "ear" else None,
                 cluster=(mean(0, 5), mean(3, 6)) if self.w.clusters else None,
                 clocks=clocks.summary())
        if self.w.mode == "structured":  # one entry per denoising step of the cycle
            by_step = {}
            for i in range(steps):
                by_step.setdefault(self.cycle[i % len(self.cycle)], []).append(per_call[i])
            r["by_step"] = {str(st): float(np.mean(v)) for st, v in sorted(by_step.items())}
        return r

    def secondary(self, steps: int):
        """World model: the frames before the chunk form a KV cache whose pooled tables carry
        over between chunks; only the chunk's own blocks are pooled (labelled row)."""
        torch, ses, A, w, op, p = self.ses.torch, self.ses, self.A, self.w, self.op, self.p
        j0 = kv_cached_start(w)
        if not j0:
            return None
        q, k, v = self.q, self.k, self.v
        A.pool(q, k, v, p, op.tables)           # the cache's tables, once
        torch.cuda.synchronize(ses.dev)
        ev2 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        ses.barrier()
        torch.cuda.synchronize(ses.dev)
        for i in range(steps):
            e = ev2[i]
            e[0].record(ses.stream)
            A.pool(q, k, v, p, op.tables, kv_block_start=j0)
            e[1].record(ses.stream)
            A.route(p, op.tables, op.kv_idx, op.kv_cnt, w.mode, w.rho, w.tau)
            e[2].record(ses.stream)
            op.forward_stage(p, op.tables, op.kv_idx, op.kv_cnt, q, k, v, op.out)
            e[3].record(ses.stream)
        torch.cuda.synchronize(ses.dev)
        ses.barrier()
        ms2 = ses.max(float(np.mean([e[0].elapsed_time(e[3]) for e in ev2])))
        m = lambda a, b: float(np.mean([e[a].elapsed_time(e[b]) for e in ev2]))
        return {"label": f"KV cache pooled once: only the chunk's blocks {j0}..{w.nkb - 1} "
                         f"pooled per call",
                "value": ses.D.weak_scaling_value(w.dense_flops(), ses.world, ms2), "unit": UNIT,
                "ms_per_step": ms2,
                "stages_ms": {"pool": m(0, 1), "route": m(1, 2), "forward": m(2, 3)}}

    def graph(self, steps: int):
        """The same steps replayed from CUDA graphs (one per denoising step of the cycle)."""
        torch, ses, op = self.ses.torch, self.ses, self.op
        graphs = {st: op.capture(self.q, self.k, self.v, step=st) for st in sorted(set(self.cycle))}
        for st in self.cycle:
            graphs[st].replay()
        torch.cuda.synchronize(ses.dev)
        ses.barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(ses.stream)
        for i in range(steps):
            graphs[self.cycle[i % len(self.cycle)]].replay()
        g1.record(ses.stream)
        torch.cuda.synchronize(ses.dev)
        ses.barrier()
        gms = ses.max(g0.elapsed_time(g1) / steps)
        del graphs
        return {"ms_per_step": gms,
                "value": ses.D.weak_scaling_value(self.w.dense_flops(), ses.world, gms),
                "unit": UNIT, "graphs": len(set(self.cycle))}

    def e2e(self, steps: int) -> dict:
        """Through the public host-buffer call: per step, Q, K, V go from pinned host memory
        to the device and the output comes back, overlapped with the compute range by range
        of heads and, across steps, with the neighbouring steps' compute."""
        torch, ses, op = self.ses.torch, self.ses, self.op
        out_h = torch.empty(op.out.shape, dtype=op.out.dtype, pin_memory=True)
        op.run_from_host(self.q_h, self.k_h, self.v_h, out_h, step=0)
        torch.cuda.synchronize(ses.dev)
        ses.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(ses.stream)
        for i in range(steps):
            op.run_from_host(self.q_h, self.k_h, self.v_h, out_h,
                             step=self.cycle[i % len(self.cycle)])
        op.wait_host_copies()   # the last output copy ends inside the timed region
        s1.record(ses.stream)
        torch.cuda.synchronize(ses.dev)
        ses.barrier()
        e2e_ms = ses.max(s0.elapsed_time(s1) / steps)
        h2d = sum(x.numel() * x.element_size() for x in (self.q_h, self.k_h, self.v_h))
        d2h = out_h.numel() * out_h.element_size()
        return {"value": ses.D.weak_scaling_value(self.w.dense_flops(), ses.world, e2e_ms),
                "unit": UNIT, "ms_per_step": e2e_ms, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)}

    def report(self, r: dict, pk: dict) -> dict:
        """Per-call figures and roofline fractions of one measured workload."""
        w, op, ses = self.w, self.op, self.ses
        kv_idx, kv_cnt = op.kv_idx.cpu().numpy(), op.kv_cnt.cpu().numpy()
        fl = executed_flops(w, kv_idx, kv_cnt)
        fwd_s = r["forward"] / 1e3
        achieved = fl["total"] / fwd_s / 1e12
        kept = fl["exact"] / fwd_s / 1e12
        pool_s = r["pool"] / 1e3
        pb = pool_bytes(w, w.mode != "structured")
        extra = pool_extra_bytes(w)
        rb, rf = route_work(w)
        route_s = r["route"] / 1e3
        out = {
            "ms_per_call": r["ms_step"],
            "ms_per_call_median": float(np.median(r["per_call"])),
            "value": ses.D.weak_scaling_value(w.dense_flops(), ses.world, r["ms_step"]),
            "unit": UNIT,
            "stages_ms": {"pool": r["pool"], "route" if w.mode != "structured" else "mask":
                          r["route"], "forward": r["forward"]},
            "roofline": {"kernel": "sparse_attn_forward", "bound": "tensor", "achieved": achieved,
                         "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_sustained"],
                         "frac_of_burst": achieved / pk["bf16"],
                         "kept_only": {"achieved": kept, "frac": kept / pk["bf16_sustained"],
                                       "frac_of_burst": kept / pk["bf16"]},
                         "traffic": forward_traffic(w),
                         "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                         "peak_kind": f"bf16 sustained ({pk['source']}); frac_of_burst against "
                                      f"the burst peak {pk['bf16']}",
                         "flops_per_launch": fl},
            "pool_roofline": {"bound": "hbm", "bytes": pb, "achieved": pb / pool_s / 1e9,
                              "peak": pk["hbm"], "unit": "GB/s",
                              "frac": pb / pool_s / 1e9 / pk["hbm"],
                              "extra_bytes": extra,
                              "frac_with_extra": (pb + sum(extra.values())) / pool_s / 1e9
                              / pk["hbm"]},
            "route_roofline": {"bound": "latency", "bytes": rb, "achieved_gbs": rb / route_s / 1e9,
                               "hbm_frac": rb / route_s / 1e9 / pk["hbm"], "fp32_flops": rf,
                               "fp32_frac": rf / route_s / 1e12 / FP32_PEAK_TFLOPS,
                               "fp32_peak_tflops": FP32_PEAK_TFLOPS},
            "clocks": r["clocks"],
            "forward_splits": op.last_splits,
        }
        if "by_step" in r:
            out["ms_per_call_by_step"] = r["by_step"]
        if r["cluster"] is not None:
            out["stages_ms"]["cluster"], out["stages_ms"]["unpermute"] = r["cluster"]
        if r["probe"] is not None:
            # the probe's algorithmic work: logits and the value product, each
            # 2 * nqb * Nk * d per head (the 2-piece splits are not counted)
            ear_fl = 4.0 * w.B * w.H * w.nqb * w.Nk * w.d
            out["stages_ms"]["ear_probe"] = r["probe"]
            out["ear_roofline"] = {"kernel": "sparse_attn_ear_scores", "bound": "tensor",
                                   "achieved": ear_fl / (r["probe"] / 1e3) / 1e12,
                                   "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                                   "frac": ear_fl / (r["probe"] / 1e3) / 1e12 / pk["bf16_sustained"],
                                   "peak_kind": f"bf16 sustained ({pk['source']})",
                                   "flops_per_launch": ear_fl}
        return out


def workload_config(w: W.Workload, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
            "block": w.block, "order": w.order, "mode": w.mode, "keep": keep_label(w),
            "output": "fp32",
            "l2": "inputs exceed L2 (Q+K+V %.2f GB per GPU)" % (
                (w.B * w.H * (w.Nq + 2 * w.Nk) * w.d * 2) / 1e9) if
            w.B * w.H * (w.Nq + 2 * w.Nk) * w.d * 2 > 126e6 else
            "inputs fit in L2 (%.1f MB): latency-bound small case" % (
                (w.B * w.H * (w.Nq + 2 * w.Nk) * w.d * 2) / 1e6),
            "parallelism": f"weak: {world} independent problems, one per GPU"}


def main():
    args = parse()
    w = W.WORKLOADS[args.workload]
    if args.heads:
        w = W.shrink(w, H=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
        return

    ses = Session()
    pk = peaks()
    b = Bench(ses, w, splits=args.splits or None)
    r = b.run(args.steps, args.warmup)
    graph = b.graph(args.steps) if args.graphs else None
    secondary = b.secondary(args.steps)
    rep = b.report(r, pk)
    e2e = None if args.no_e2e else b.e2e(args.e2e_steps)
    launches = launches_per_step(w, b.op.last_splits) * args.steps
    del b

    # The other configurations of the benchmark set, each measured the same way in this
    # run (one GPU only: every rank would otherwise generate every workload's inputs).
    others = {}
    if ses.world == 1 and not args.no_workloads and w.name == W.METRIC_WORKLOAD:
        for name in OTHER_CONFIGS:
            wo = W.WORKLOADS[name]
            bo = Bench(ses, wo)
            steps = max(args.steps, len(bo.cycle))
            ro = bo.run(steps, max(args.warmup, 3))
            entry = {"config": workload_config(wo, ses.world), "steps": steps,
                     "warmup": max(args.warmup, 3), **bo.report(ro, pk)}
            sec = bo.secondary(steps)
            if sec is not None:
                entry["secondary"] = sec
            launches += launches_per_step(wo, bo.op.last_splits) * steps
            others[name] = entry
            del bo
            ses.torch.cuda.empty_cache()

    cpu = None
    if ses.rank == 0 and ses.world == 1 and not args.no_cpu_baseline:
        res = time_oracle(w, args.cpu_seconds)
        cpu = {k: res[k] for k in ("value", "unit", "cores", "cpu_count", "blas", "kind", "sample")}

    if ses.rank == 0:
        value = ses.D.weak_scaling_value(w.dense_flops(), ses.world, r["ms_step"])
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ses.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(w, ses.world),
            "pct_of_bf16_peak_dense_equiv": 100.0 * value / ses.world / pk["bf16"],
            "stages_ms": rep["stages_ms"], "roofline": rep["roofline"],
            "pool_roofline": rep["pool_roofline"], "route_roofline": rep["route_roofline"],
            "clocks": rep["clocks"], "gpu_launches": launches,
            "forward_splits": rep["forward_splits"], "e2e": e2e, "cpu_baseline": cpu,
            "ms_per_call_median": rep["ms_per_call_median"],
        }
        for key in ("ms_per_call_by_step", "ear_roofline"):
            if key in rep:
                line[key] = rep[key]
        if secondary is not None:
            line["secondary"] = secondary
        if graph is not None:
            line["graph"] = graph
        if w.clusters:
            line["config"]["clusters"] = {"C_q": w.clusters[0], "C_k": w.clusters[1],
                                          "iters": w.clusters[2]}
        if others:
            line["workloads"] = others
        print(json.dumps(line), flush=True)
    if ses.world > 1:
        import torch.distributed as tdist
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()
