"""The C ABI library loads, exports every entry point the header declares, and
rejects bad arguments on the host (no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

from free_block_sparse_kv_b200 import build
from free_block_sparse_kv_b200 import sparse_attn as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sparse_attn_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return C.load_library()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared >= set(C.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_table_sizes():
    assert C.sparse_attn_table_sizes(1, 40, 75600, 75600, 128, 128, 1) == (
        40 * 591 * 128 * 4, 40 * 591 * 128 * 4, 40 * 591 * 128 * 4,
        40 * 2 * 591 * 128 * 2, 40 * 591 * 128 * 2, 40 * 591 * 128 * 128 * 2, 40 * 75600 * 128 * 2)
    assert C.sparse_attn_table_sizes(4, 16, 1560, 63960, 128, 64, 0)[5] == 0
    assert C.sparse_attn_table_sizes(4, 16, 1560, 63960, 128, 64, 2)[5] == 4 * 16 * 1000 * 128 * 128 * 2
    assert C.sparse_attn_table_sizes(4, 16, 1560, 63960, 128, 64, 0)[0] == 4 * 16 * 25 * 128 * 4
    cent, cw, iw = C.sparse_attn_kmeans_sizes(1, 40, 75600, 128, 296)
    assert cent == 40 * 296 * 128 * 8
    assert cw >= 40 * 2 * 384 * 128 * 2 + 40 * 384 * 4      # padded bf16 pieces, norms
    assert iw >= 40 * 74 * 296 * 4 + 40 * 75600 * 4 + 40 * 4


def test_host_argument_checks(lib):
    buf = (ctypes.c_char * 4096)()
    base = ctypes.addressof(buf)
    p = base + (-base) % 16
    cases = [
        lambda: C.sparse_attn_table_sizes(1, 1, 64, 64, 96, 64, 0),
        lambda: C.sparse_attn_table_sizes(1, 1, 64, 64, 64, 32, 0),
        lambda: C.sparse_attn_table_sizes(-1, 1, 64, 64, 64, 64, 0),
        lambda: C.sparse_attn_pool(p, p, p, 1, 1, 64, 64, 64, 64, 3, p, p, p, p, p, p, p, None, 0),
        lambda: C.sparse_attn_pool(p, p, p, 1, 1, 64, 64, 64, 64, 2, p, p, p, p, p, None, p, None, 0),
        lambda: C.sparse_attn_pool(p, None, p, 1, 1, 64, 64, 64, 64, 0, p, p, p, p, p, None, p, None, 0),
        lambda: C.sparse_attn_pool(p, p + 8, p, 1, 1, 64, 64, 64, 64, 0, p, p, p, p, p, None, p, None, 0),
        lambda: C.sparse_attn_pool(p, p, p, 1, 1, 64, 64, 64, 64, 0, p, p, p, p, p, None, None, None, 0),
        lambda: C.sparse_attn_pool(p, p, p, 1, 1, 64, 64, 64, 64, 0, p, p, p, p, p, None, p, p + 2, 0),
        lambda: C.sparse_attn_route(p, p, 1, 1, 4, 3000, 64, 0, 1, 4, 0.9, 0.1, p, p, 750, 0),
        lambda: C.sparse_attn_route(p, p, 1, 1, 4, 10, 64, 0, 3, 2, 0.9, 0.1, p, p, 10, 0),
        lambda: C.sparse_attn_route(p, p, 1, 1, 4, 10, 64, 1, 1, 4, 1.5, 0.1, p, p, 10, 0),
        lambda: C.sparse_attn_route(p, p, 1, 1, 4, 10, 64, 7, 1, 4, 0.9, 0.1, p, p, 10, 0),
        lambda: C.sparse_attn_route_cov(p, p, None, 1, 1, 4, 10, 64, 1, 4, 0.1, p, p, 10, 0),
        lambda: C.sparse_attn_route_cov(p, p, p, 1, 1, 4, 10, 64, 1, 4, 0.1, p, p, 2, 0),
        lambda: C.sparse_attn_route_cov(p, p, p, 1, 1, 4, 10, 96, 1, 4, 0.1, p, p, 10, 0),
        lambda: C.sparse_attn_hbar(p, 1, 1, 4, 96, p, p, p, 0),
        lambda: C.sparse_attn_hbar(None, 1, 1, 4, 64, p, p, p, 0),
        lambda: C.sparse_attn_hbar(p, 1, 1, 4, 64, p, None, p, 0),
        lambda: C.sparse_attn_hbar(p, 1, 1, 0, 64, p, p, p, 0),
        lambda: C.sparse_attn_forward(p, p, p, p, p, None, p, p, 1, 1, 1, 64, 64, 64, 64, 2, 0.1, p,
                                      0, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 640, 96, 64, 0.1, p, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 640, 64, 32, 0.1, p, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p + 8, p, 1, 1, 4, 640, 64, 64, 0.1, p, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 640, 64, 64, 0.1, None, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 640, 64, 64, 0.1, p + 2, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 640, 64, 64, float("inf"), p, None, 0),
        lambda: C.sparse_attn_ear_scores(p, p, p, 1, 1, 4, 64 * 4096, 64, 64, 0.1, p, None, 0),
        lambda: C.sparse_attn_route_scores(p, 1, 1, 4, 10, 1, 4, p, p, 2, 0),
        lambda: C.sparse_attn_route_scores(p, 1, 1, 4, 10, 5, 4, p, p, 10, 0),
        lambda: C.sparse_attn_route_scores(None, 1, 1, 4, 10, 1, 4, p, p, 10, 0),
        lambda: C.sparse_attn_route_scores(p, 1, 1, 4, 0, 1, 4, p, p, 10, 0),
        lambda: C.sparse_attn_pool_incremental(p, p, p, 1, 1, 64, 640, 64, 64, 0, 11, p, p, p, p,
                                               p, None, p, None, 0),
        lambda: C.sparse_attn_pool_incremental(p, p, p, 1, 1, 64, 640, 64, 64, 1, 2, p, p, p, p,
                                               p, None, p, None, 0),
        lambda: C.sparse_attn_wait_selftest(p, 0, p, 0),
        lambda: C.sparse_attn_wait_selftest(None, 10, p, 0),
        lambda: C.sparse_attn_kmeans_sizes(1, 1, 64, 96, 4),
        lambda: C.sparse_attn_kmeans_sizes(1, 1, 64, 64, 0),
        lambda: C.sparse_attn_kmeans_sizes(1, 1, 64, 64, 5000),
        lambda: C.sparse_attn_kmeans(p, 1, 1, 64, 64, 65, 2, p, p, p, p, p, p, None, 0),
        lambda: C.sparse_attn_kmeans(p, 1, 1, 64, 64, 4, -1, p, p, p, p, p, p, None, 0),
        lambda: C.sparse_attn_kmeans(p + 8, 1, 1, 64, 64, 4, 2, p, p, p, p, p, p, None, 0),
        lambda: C.sparse_attn_kmeans(p, 1, 1, 64, 64, 4, 2, p, None, p, p, p, p, None, 0),
        lambda: C.sparse_attn_permute_rows(p, p, 1, 1, 64, 100, 1, p + 16, 0),
        lambda: C.sparse_attn_permute_rows(p, p, 1, 1, 64, 128, 2, p + 16, 0),
        lambda: C.sparse_attn_permute_rows(p, p, 1, 1, 64, 128, 1, p, 0),
        lambda: C.sparse_attn_structured_mask(1, 1, 64, 6400, 64, 10, 10, 1, 1, 1, 0, 0, p, p, 100, 0),
        lambda: C.sparse_attn_structured_mask(1, 1, 64, 64, 64, 8, 8, 1, 1, 0, 0, 0, p, p, 1, 0),
        lambda: C.sparse_attn_structured_mask_adaptive(1, 1, 64, 64, 64, 8, 8, 1, 1, 2, 0, 0, -1, p,
                                                       p, 1, 0),
        lambda: C.sparse_attn_forward(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 0, 64, 64, 0, 0.1, p, 0,
                                      None, 0),
        lambda: C.sparse_attn_forward(p, p, p, p, p, None, p, p, 1, 1, 1, 64, 64, 64, 64, 1, 0.1, p,
                                      0, None, 0),
        lambda: C.sparse_attn_forward(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 64, 64, 0, 0.1, p, 5,
                                      None, 0),
        lambda: C.sparse_attn_forward(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64 * 4096, 64, 64, 0, 0.1,
                                      p, 0, None, 0),
        lambda: C.sparse_attn_forward_split(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 64, 64, 0, 0.1,
                                            0, p, p, 0, None, 0),
        lambda: C.sparse_attn_forward_split(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 64, 64, 0, 0.1,
                                            17, p, p, 0, None, 0),
        lambda: C.sparse_attn_forward_split(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 64, 64, 0, 0.1,
                                            2, None, p, 0, None, 0),
        lambda: C.sparse_attn_forward_split(p, p, p, p, p, p, p, p, 1, 1, 1, 64, 64, 64, 64, 0, 0.1,
                                            2, p + 4, p, 0, None, 0),
        lambda: C.sparse_attn_forward_work_bytes(1, 1, 64, 64, 0),
        lambda: C.sparse_attn_forward_split_plan(1, 1, 64, 64, 64, 64, -1),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(C.SparseAttnError) as e:
            call()
        assert e.value.code == C.SA_ERR_INVALID, (i, str(e.value))
        assert C.sparse_attn_last_error(), i


def test_split_plan_on_the_host(lib):
    """The split choice for a given SM count (no device needed): no split where the grid
    spans many waves or the keys form one run of 64 blocks; a split of the world-model
    chunk whose modelled schedule beats the unsplit one; scratch as documented."""
    assert C.sparse_attn_forward_split_plan(1, 40, 75600, 75600, 128, 128, 148) == (1, 0)
    assert C.sparse_attn_forward_split_plan(1, 2, 4096, 4096, 128, 64, 148) == (1, 0)
    assert C.sparse_attn_forward_split_plan(1, 2, 0, 4096, 128, 64, 148) == (1, 0)
    n, b = C.sparse_attn_forward_split_plan(4, 16, 1560, 63960, 128, 64, 148)
    assert 2 <= n <= 16 and b == n * 4 * 16 * 1560 * (128 + 2) * 4
    # a single (batch, head) with 16 runs of 64 blocks: 7 CTAs on 148 SMs split far
    n1, _ = C.sparse_attn_forward_split_plan(1, 1, 1560, 63960, 128, 64, 148)
    assert 8 <= n1 <= 16
    # never more splits than runs of 64 blocks
    n2, _ = C.sparse_attn_forward_split_plan(1, 1, 1560, 3 * 64 * 64, 128, 64, 148)
    assert n2 <= 3
    assert C.sparse_attn_forward_work_bytes(2, 3, 100, 64, 1) == 0
    assert C.sparse_attn_forward_work_bytes(2, 3, 100, 64, 4) == 4 * 2 * 3 * 100 * 66 * 4


def test_binding_fails_loudly_without_library(tmp_path):
    saved = C._lib
    C._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            C.load_library(str(tmp_path / "absent.so"))
    finally:
        C._lib = saved
