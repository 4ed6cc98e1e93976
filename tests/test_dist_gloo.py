"""The multi-process path of the benchmark on CPU: two gloo ranks, launched like
torchrun would (RANK / WORLD_SIZE / MASTER_* in the environment). Checks the
rank-seeded workloads (same shapes, different draws), the max-over-ranks timing and
the whole-job throughput the rank-0 line reports."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from free_block_sparse_kv_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from free_block_sparse_kv_b200 import dist as D
    assert D.env_ranks() == (world, rank, rank)
    D.init("gloo", timeout_s=60)
    w = D.rank_workload(W.WORKLOADS["uniform-4k"], rank)
    q, k, v = W.head_inputs_bits(W.shrink(w, Nq=256, Nk=256), 0, 0)
    D.barrier()
    ms = 10.0 + 5.0 * rank                   # the slower rank must win
    ms_max = D.max_over_ranks(ms)
    value = D.weak_scaling_value(1e12, world, ms_max)
    out.put((rank, w.seed, q.tobytes(), ms_max, value))
    import torch.distributed as tdist
    tdist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, q0, m0, v0), (r1, s1, q1, m1, v1) = res
    assert (r0, r1) == (0, 1) and s0 != s1
    assert q0 != q1 and len(q0) == len(q1)           # same shapes, different draws
    assert m0 == m1 == 15.0                           # max over ranks
    assert np.isclose(v0, 2 * 1e12 / 0.015 / 1e12) and v0 == v1


def test_single_process_helpers_are_identity():
    from free_block_sparse_kv_b200 import dist as D
    assert D.max_over_ranks(3.5) == 3.5
    assert D.rank_workload(W.WORKLOADS["uniform-4k"], 0).seed == W.WORKLOADS["uniform-4k"].seed
