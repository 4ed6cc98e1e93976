"""The k-means entry point without caller scratch: same results as the entry point that
takes scratch buffers (bit for bit), and problems larger than its built-in buffer are
rejected on the host. Collected last, so that the built-in buffer is first touched after
every other test has run."""
import numpy as np
import pytest
import torch

from free_block_sparse_kv_b200 import attention as A
from free_block_sparse_kv_b200 import build
from free_block_sparse_kv_b200 import sparse_attn as C
from free_block_sparse_kv_b200 import workloads as W


def test_oversized_problem_is_rejected_on_the_host():
    build.build()
    C.load_library()
    # 40 heads x 300,000 tokens: the sorting and candidate lists alone exceed 32 MiB
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_kmeans_noalloc(16, 1, 40, 300000, 128, 296, 3, 16, 16, 16, 16, None, 0)
    assert e.value.code == C.SA_ERR_INVALID and "scratch" in str(e.value)


def _a256(x):
    return -(-x // 256) * 256


@pytest.mark.parametrize("B,H,N,d,C_", [(1, 2, 3000, 64, 130), (1, 40, 75600, 128, 296),
                                        (4, 16, 63960, 128, 250), (2, 3, 1, 64, 1)])
def test_scratch_sizes_cover_every_work_buffer(B, H, N, d, C_):
    """sizes[1] and sizes[2] are the ends of the work buffers the launcher carves out of
    cwork and iwork: padded centroid pieces, their norms, fp64 segment sums; per-chunk
    histograms, the near-tie list, its count and the segment offsets (each 256-byte
    aligned but the last)."""
    build.build()
    C.load_library()
    bh = B * H
    cpad = -(-C_ // 128) * 128
    nchunk, maxseg = -(-N // 1024), -(-N // 512) + C_
    cw = _a256(bh * 2 * cpad * d * 2) + _a256(bh * cpad * 4) + bh * maxseg * d * 8
    iw = _a256(bh * nchunk * C_ * 4) + _a256(bh * N * 4) + _a256(bh * 4) + bh * (C_ + 1) * 4
    assert C.sparse_attn_kmeans_sizes(B, H, N, d, C_) == (bh * C_ * d * 8, cw, iw)


def test_the_largest_problems_that_fit_and_the_first_that_does_not():
    """32 heads of 75,600 tokens with 296 clusters need just under 32 MiB of scratch; 33
    heads need just over it and are rejected before anything reaches the device."""
    build.build()
    C.load_library()
    need = lambda H: _a256(C.sparse_attn_kmeans_sizes(1, H, 75600, 128, 296)[1]) + \
        C.sparse_attn_kmeans_sizes(1, H, 75600, 128, 296)[2]
    assert need(32) <= 32 << 20 < need(33)
    with pytest.raises(C.SparseAttnError) as e:
        C.sparse_attn_kmeans_noalloc(16, 1, 33, 75600, 128, 296, 3, 16, 16, 16, 16, None, 0)
    assert e.value.code == C.SA_ERR_INVALID and "scratch" in str(e.value)


@pytest.mark.gpu
@pytest.mark.parametrize("d,N,C_,iters,H", [(64, 3000, 130, 2, 2), (128, 9480, 38, 3, 2),
                                            (128, 75600, 296, 1, 32)])
def test_noalloc_equals_the_scratch_entry_point(d, N, C_, iters, H):
    """Two calls in a row equal the scratch entry point bit for bit, on small problems and
    on one that fills the built-in buffer to within 1% (32 heads of 75,600 tokens)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    B = 1
    rng = np.random.default_rng(60 + d)
    bits = W.bf16_round(rng.standard_normal((B, H, N, d)).astype(np.float32))[1]
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    ref = A.allocate_clustering(B, H, N, d, C_, iters, "cuda")
    A.kmeans(x, ref)
    i32 = dict(dtype=torch.int32, device="cuda")
    cent = torch.empty(B, H, C_, d, dtype=torch.float64, device="cuda")
    labels, perm = torch.empty(B, H, N, **i32), torch.empty(B, H, N, **i32)
    offsets = torch.empty(B, H, C_ + 1, **i32)
    flag = torch.zeros(1, **i32)
    for _ in range(2):  # the shared buffer is reused call after call
        C.sparse_attn_kmeans_noalloc(x, B, H, N, d, C_, iters, cent, labels, perm, offsets, flag)
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        assert torch.equal(labels, ref.labels) and torch.equal(perm, ref.perm)
        assert torch.equal(offsets, ref.offsets) and torch.equal(cent, ref.centroids)
