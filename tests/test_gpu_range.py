"""Large values through the fp16 tables of the pool.

The pool writes the value sums S_j, the first-order matrices M_j and a copy of V in fp16
(the forward multiplies them by fp16 probabilities on the tensor cores). Inputs whose
tables fit in fp16 must still match the oracle (PISA §2 "Algorithme Central": N_t and D_t
are defined for any input); inputs whose tables do not fit must be reported (SA_ERR_RANGE),
never turned silently into infinities.
"""
import dataclasses

import numpy as np
import pytest
import torch

from free_block_sparse_kv_b200 import attention as A
from free_block_sparse_kv_b200 import sparse_attn as C
from free_block_sparse_kv_b200 import workloads as W
from oracle import block_sparse_attention as O
from tests.helpers import MEAN_REL, SMALL, err_stats

pytestmark = pytest.mark.gpu

# The reduced 720p case with key outliers scaled x10 instead of x4.
BASE = dataclasses.replace(SMALL["dit720p-small"], name="dit720p-small-outliers10",
                           outlier_scale=10.0)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _inputs(v_scale):
    """Q, K as drawn; V drawn then scaled by v_scale and rounded to bf16 (bit patterns)."""
    qb, kb, vb = W.full_inputs_bits(BASE)
    v = W.bits_to_f32(vb) * np.float32(v_scale)
    return qb, kb, W.bf16_round(v)[1]


def _op():
    p = A.Problem(BASE.B, BASE.H, BASE.Nq, BASE.Nk, BASE.d, BASE.block, BASE.order)
    return A.BlockSparseAttention(p, "topk", rho=BASE.rho)


def test_values_of_a_few_hundred_match_the_oracle():
    """V ~ 100 N(0,1) with keys x10 outliers: M_j reaches ~24,000, within fp16. Outputs
    within max abs 1e-2 max|V| and mean relative 2e-3 of the oracle on sampled rows."""
    qb, kb, vb = _inputs(100.0)
    op = _op()
    out = op(_dev(qb), _dev(kb), _dev(vb))
    torch.cuda.synchronize()
    op.check()
    got = out.cpu().numpy()
    rows = np.arange(0, BASE.Nq, 7)
    for h in range(BASE.H):
        q, k, v = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        kept = O.route_head(q, k, BASE.block, "topk", BASE.scale, keep=BASE.keep())[0]
        want = O.forward_head(q, k, v, kept, BASE.block, BASE.order, BASE.scale, rows=rows)
        mx, rel = err_stats(got[0, h, rows], want)
        assert mx <= 1e-2 * np.abs(v).max() and rel <= MEAN_REL, (h, mx, rel)


@pytest.mark.parametrize("case", ["M_j above 65504", "one value above 65504"])
def test_tables_outside_fp16_are_reported(case):
    if case == "M_j above 65504":
        qb, kb, vb = _inputs(300.0)   # M_j reaches ~72,500
    else:
        qb, kb, vb = _inputs(1.0)
        v = W.bits_to_f32(vb)
        v[0, 1, 4321, 17] = 70000.0   # bf16 69,632: rounds to infinity in fp16
        vb = W.bf16_round(v)[1]
    op = _op()
    op(_dev(qb), _dev(kb), _dev(vb))
    torch.cuda.synchronize()
    assert int(op.err_flag.item()) & C.SA_FLAG_RANGE
    with pytest.raises(C.SparseAttnError) as e:
        op.check()
    assert e.value.code == C.SA_ERR_RANGE
    # the flag is sticky until cleared; the context stays usable for the next call
    op.err_flag.zero_()
    qb, kb, vb = _inputs(1.0)
    op(_dev(qb), _dev(kb), _dev(vb))
    torch.cuda.synchronize()
    op.check()
