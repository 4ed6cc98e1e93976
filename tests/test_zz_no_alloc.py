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


@pytest.mark.gpu
@pytest.mark.parametrize("d,N,C_,iters", [(64, 3000, 130, 2), (128, 9480, 38, 3)])
def test_noalloc_equals_the_scratch_entry_point(d, N, C_, iters):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    B, H = 1, 2
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
