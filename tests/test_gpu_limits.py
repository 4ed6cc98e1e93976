"""The largest problems the library accepts: SA_MAX_KV_BLOCKS key blocks per head.

At 2048 key blocks the route holds 64 score keys per lane and the forward's kept bitmaps
use all of their words; block 64 (the world-model blocking) puts that at 131,072 keys.
Masks bit-exact above the gate and outputs within the usual bar against the oracle, on a
ragged query chunk, for top-k and covering-mass routing and both compensation orders.
One past the limit is rejected on the host.
"""
import ctypes

import numpy as np
import pytest
import torch

from free_block_sparse_kv_b200 import attention as A
from free_block_sparse_kv_b200 import sparse_attn as C
from free_block_sparse_kv_b200 import workloads as W
from oracle import block_sparse_attention as O
from tests.helpers import GATE, MAX_ABS, MEAN_REL, err_stats, lists_to_sets

MAX_NKB = 2048


def test_one_block_past_the_limit_is_rejected_on_the_host():
    C.load_library()
    buf = (ctypes.c_char * 4096)()
    base = ctypes.addressof(buf)
    p = base + (-base) % 16
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_route(p, p, 1, 1, 4, MAX_NKB + 1, 64, 0, 1, 10, 0.9, 0.1, p, p, 300, 0)
    assert e.value.code == C.SA_ERR_INVALID
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_forward(p, p, p, p, p, None, p, p, 10, 1, 1, 64, 64 * (MAX_NKB + 1), 64, 64,
                              0, 0.1, p, 0, None, 0)
    assert e.value.code == C.SA_ERR_INVALID


@pytest.mark.gpu
@pytest.mark.parametrize("mode,order", [("topk", 0), ("mass", 1)])
def test_maximum_key_blocks(mode, order):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()
    block, d = 64, 128
    w = W.shrink(W.WORKLOADS["worldmodel-chunk"], name="max-kv-blocks", B=1, H=1, Nq=300,
                 Nk=MAX_NKB * block, grid=(85, 30, 52), q_frame0=83, order=order, mode=mode,
                 rho=(1, 10), block=block, d=d)
    assert w.nkb == MAX_NKB
    qb, kb, vb = W.full_inputs_bits(w)
    dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()
    op = A.BlockSparseAttention(A.Problem(w.B, w.H, w.Nq, w.Nk, w.d, w.block, w.order), mode,
                                rho=w.rho, tau=w.tau)
    out = op(dev(qb), dev(kb), dev(vb))
    torch.cuda.synchronize()
    op.check()
    q, k, v = (W.bits_to_f32(x[0, 0]) for x in (qb, kb, vb))
    kept, s, counts = O.route_head(q, k, block, mode, w.scale, keep=w.keep(), tau=w.tau)
    gaps, lo, hi = O.gate_diagnostics(s, counts, tau=w.tau if mode == "mass" else None)
    gate = gaps > GATE if mode == "topk" else (gaps > GATE) & (lo > GATE) & (hi > GATE)
    got = lists_to_sets(op.kv_idx[0, 0].cpu().numpy(), op.kv_cnt[0, 0].cpu().numpy())
    for i in range(w.nqb):
        if gate[i]:
            assert got[i] == kept[i].tolist(), (mode, i)
    rows = np.array([0, 1, 63, 64, 150, 255, 256, w.Nq - 1])
    want = O.forward_head(q, k, v, kept, block, order, w.scale, rows=rows)
    mx, mr = err_stats(out[0, 0, rows].cpu().numpy(), want)
    assert mx <= MAX_ABS and mr <= MEAN_REL, (mode, mx, mr)
