"""The seeded input generator shared by the oracle and the CUDA path (CPU only).

A slip here would feed both sides the same wrong inputs, which no parity test can see, so the
rounding is pinned against torch's own fp32 -> bf16 conversion and the draws against their
stated seeding."""
import numpy as np
import torch

from free_block_sparse_kv_b200 import dist as D
from free_block_sparse_kv_b200 import workloads as W
from tests.helpers import SMALL


def test_bf16_round_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 10000),
        # exact halfway points between two bf16 values, both parities of the lower one
        ((np.arange(1, 2001, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)).view(np.float32),
        -((np.arange(1, 2001, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.0e38, 1.0, -1.0], np.float32),
    ]).astype(np.float32)
    vals, bits = W.bf16_round(x)
    want = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(bits.view(np.int16), want.view(torch.int16).numpy())
    assert np.array_equal(vals, want.float().numpy())
    assert np.array_equal(W.bits_to_f32(bits), vals)


def test_draws_are_reproducible_and_thread_independent():
    w = SMALL["worldmodel-small"]
    a = W.head_inputs_bits(w, 1, 0)
    b = W.head_inputs_bits(w, 1, 0)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    one = W.full_inputs_bits(w, threads=1)
    many = W.full_inputs_bits(w, threads=4)
    assert all(np.array_equal(x, y) for x, y in zip(one, many))
    assert all(np.array_equal(full[1, 0], head) for full, head in zip(one, a))


def test_heads_tensors_and_ranks_draw_different_numbers():
    w = SMALL["dit-small"]
    q0, k0, v0 = W.head_inputs(w, 0, 0)
    q1, _, _ = W.head_inputs(w, 0, 1)
    assert not np.array_equal(q0, q1)
    assert not np.array_equal(q0[:100], k0[:100])
    r1 = W.head_inputs(D.rank_workload(w, 1), 0, 0)
    assert not np.array_equal(r1[2], v0)
    assert np.array_equal(W.head_inputs(D.rank_workload(w, 0), 0, 0)[2], v0)


def test_shapes_and_structure_of_the_recipes():
    for name, w in SMALL.items():
        q, k, v = W.head_inputs(w, 0, 0)
        assert q.shape == (w.Nq, w.d) and k.shape == (w.Nk, w.d) and v.shape == (w.Nk, w.d), name
        assert np.isfinite(q).all() and np.isfinite(k).all() and np.isfinite(v).all(), name
    # patch recipe: keys of one spatio-temporal patch share a centre, so they sit much closer
    # to each other than to keys of other patches
    w = SMALL["dit-small"]
    _, k, _ = W.head_inputs(w, 0, 0)
    ids, _ = W._patch_ids(w, 0, w.Nk)
    same = ids[:400, None] == ids[None, :400]
    kk = k[:400]
    dist2 = ((kk[:, None, :] - kk[None, :, :]) ** 2).sum(-1)
    assert dist2[same].mean() < 0.25 * dist2[~same].mean()
