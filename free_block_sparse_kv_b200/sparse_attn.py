"""ctypes binding of ``libsparse_attn.so``: the C entry points under the same names.

Argument marshalling only: tensors become their data pointers, the stream
defaults to torch's current stream, and a non-zero status raises
:class:`SparseAttnError` with the library's message. Every step of the
computation runs in the library's CUDA kernels; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsparse_attn.so")

SA_OK, SA_ERR_INVALID, SA_ERR_LAUNCH, SA_ERR_TIMEOUT, SA_ERR_UNSUPPORTED, SA_ERR_RANGE = range(6)
SA_FLAG_RANGE = 1 << 20   # err_flag bit: a pooled fp16 table value did not fit
SA_ROUTE_TOPK, SA_ROUTE_MASS = 0, 1
SA_OUT_F32, SA_OUT_BF16 = 0, 1

# Entry points declared in include/sparse_attn.h.
EXPORTS = ("sparse_attn_table_sizes", "sparse_attn_pool", "sparse_attn_pool_incremental",
           "sparse_attn_route",
           "sparse_attn_route_cov", "sparse_attn_hbar", "sparse_attn_structured_mask",
           "sparse_attn_structured_mask_adaptive", "sparse_attn_ear_scores",
           "sparse_attn_route_scores", "sparse_attn_kmeans_sizes", "sparse_attn_kmeans",
           "sparse_attn_permute_rows", "sparse_attn_kmeans_noalloc", "sparse_attn_wait_selftest",
           "sparse_attn_forward", "sparse_attn_forward_split", "sparse_attn_forward_work_bytes",
           "sparse_attn_forward_split_plan", "sparse_attn_last_error")


class SparseAttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"sparse_attn error {code}: {message}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m free_block_sparse_kv_b200.build`")
    lib = ctypes.CDLL(path)
    lib.sparse_attn_last_error.restype = ctypes.c_char_p
    lib.sparse_attn_last_error.argtypes = []
    lib.sparse_attn_table_sizes.argtypes = [_I] * 7 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.sparse_attn_pool.argtypes = [_P, _P, _P] + [_I] * 7 + [_P] * 8 + [_P]
    lib.sparse_attn_pool_incremental.argtypes = [_P, _P, _P] + [_I] * 8 + [_P] * 8 + [_P]
    lib.sparse_attn_route.argtypes = [_P, _P] + [_I] * 8 + [_F, _F, _P, _P, _I, _P]
    lib.sparse_attn_route_cov.argtypes = [_P, _P, _P] + [_I] * 7 + [_F, _P, _P, _I, _P]
    lib.sparse_attn_hbar.argtypes = [_P] + [_I] * 4 + [_P, _P, _P, _P]
    lib.sparse_attn_ear_scores.argtypes = [_P, _P, _P] + [_I] * 6 + [_F, _P, _P, _P]
    lib.sparse_attn_route_scores.argtypes = [_P] + [_I] * 6 + [_P, _P, _I, _P]
    lib.sparse_attn_kmeans_sizes.argtypes = [_I] * 5 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.sparse_attn_kmeans.argtypes = [_P] + [_I] * 6 + [_P] * 7 + [_P]
    lib.sparse_attn_permute_rows.argtypes = [_P, _P] + [_I] * 5 + [_P, _P]
    lib.sparse_attn_kmeans_noalloc.argtypes = [_P] + [_I] * 6 + [_P] * 5 + [_P]
    lib.sparse_attn_wait_selftest.argtypes = [_P, _I, _P, _P]
    lib.sparse_attn_structured_mask.argtypes = [_I] * 12 + [_P, _P, _I, _P]
    lib.sparse_attn_structured_mask_adaptive.argtypes = [_I] * 13 + [_P, _P, _I, _P]
    lib.sparse_attn_forward.argtypes = [_P] * 8 + [_I] * 8 + [_F, _P, _I, _P, _P]
    lib.sparse_attn_forward_split.argtypes = [_P] * 8 + [_I] * 8 + [_F, _I, _P, _P, _I, _P, _P]
    lib.sparse_attn_forward_work_bytes.argtypes = [_I] * 5 + [ctypes.POINTER(ctypes.c_size_t)]
    lib.sparse_attn_forward_split_plan.argtypes = [_I] * 7 + [ctypes.POINTER(_I),
                                                              ctypes.POINTER(ctypes.c_size_t)]
    for name in EXPORTS[:-1]:
        getattr(lib, name).restype = _I
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != SA_OK:
        raise SparseAttnError(rc, load_library().sparse_attn_last_error().decode())


def sparse_attn_table_sizes(B, H, Nq, Nk, d, block, order):
    """Byte sizes (qbar, kbar_t, vsum, kbar16, vsum16, M, v16) of the pooled tables."""
    out = (ctypes.c_size_t * 7)()
    _check(load_library().sparse_attn_table_sizes(B, H, Nq, Nk, d, block, order, out))
    return tuple(int(x) for x in out)


def sparse_attn_pool(q, k, v, B, H, Nq, Nk, d, block, order, qbar, kbar_t, vsum, kbar16, vsum16, M,
                     v16, err_flag=None, stream=None):
    _check(load_library().sparse_attn_pool(
        _ptr(q), _ptr(k), _ptr(v), B, H, Nq, Nk, d, block, order, _ptr(qbar), _ptr(kbar_t),
        _ptr(vsum), _ptr(kbar16), _ptr(vsum16), _ptr(M), _ptr(v16), _ptr(err_flag),
        _stream(stream)))


def sparse_attn_pool_incremental(q, k, v, B, H, Nq, Nk, d, block, order, kv_block_start, qbar,
                                 kbar_t, vsum, kbar16, vsum16, M, v16, err_flag=None, stream=None):
    _check(load_library().sparse_attn_pool_incremental(
        _ptr(q), _ptr(k), _ptr(v), B, H, Nq, Nk, d, block, order, kv_block_start, _ptr(qbar),
        _ptr(kbar_t), _ptr(vsum), _ptr(kbar16), _ptr(vsum16), _ptr(M), _ptr(v16), _ptr(err_flag),
        _stream(stream)))


def sparse_attn_route(qbar, kbar_t, B, H, nqb, nkb, d, mode, rho_num, rho_den, tau, scale, kv_idx,
                      kv_cnt, cap, stream=None):
    _check(load_library().sparse_attn_route(
        _ptr(qbar), _ptr(kbar_t), B, H, nqb, nkb, d, mode, rho_num, rho_den, tau, scale,
        _ptr(kv_idx), _ptr(kv_cnt), cap, _stream(stream)))


def sparse_attn_route_cov(qbar, kbar_t, cov, B, H, nqb, nkb, d, rho_num, rho_den, scale, kv_idx,
                          kv_cnt, cap, stream=None):
    _check(load_library().sparse_attn_route_cov(
        _ptr(qbar), _ptr(kbar_t), _ptr(cov), B, H, nqb, nkb, d, rho_num, rho_den, scale,
        _ptr(kv_idx), _ptr(kv_cnt), cap, _stream(stream)))


def sparse_attn_hbar(M, B, H, nkb, d, hbar, hbar16, cov, stream=None):
    _check(load_library().sparse_attn_hbar(
        _ptr(M), B, H, nkb, d, _ptr(hbar), _ptr(hbar16), _ptr(cov), _stream(stream)))


def sparse_attn_ear_scores(qbar, k, v, B, H, nqb, Nk, d, block, scale, scores, err_flag=None,
                           stream=None):
    _check(load_library().sparse_attn_ear_scores(
        _ptr(qbar), _ptr(k), _ptr(v), B, H, nqb, Nk, d, block, scale, _ptr(scores),
        _ptr(err_flag), _stream(stream)))


def sparse_attn_route_scores(scores, B, H, nqb, nkb, rho_num, rho_den, kv_idx, kv_cnt, cap,
                             stream=None):
    _check(load_library().sparse_attn_route_scores(
        _ptr(scores), B, H, nqb, nkb, rho_num, rho_den, _ptr(kv_idx), _ptr(kv_cnt), cap,
        _stream(stream)))


def sparse_attn_kmeans_sizes(B, H, N, d, C):
    """Byte sizes (centroids, cwork, iwork) of sparse_attn_kmeans's buffers."""
    out = (ctypes.c_size_t * 3)()
    _check(load_library().sparse_attn_kmeans_sizes(B, H, N, d, C, out))
    return tuple(int(x) for x in out)


def sparse_attn_kmeans(x, B, H, N, d, C, iters, centroids, cwork, iwork, labels, perm, offsets,
                       err_flag=None, stream=None):
    _check(load_library().sparse_attn_kmeans(
        _ptr(x), B, H, N, d, C, iters, _ptr(centroids), _ptr(cwork), _ptr(iwork), _ptr(labels),
        _ptr(perm), _ptr(offsets), _ptr(err_flag), _stream(stream)))


def sparse_attn_kmeans_noalloc(x, B, H, N, d, C, iters, centroids, labels, perm, offsets,
                               err_flag=None, stream=None):
    _check(load_library().sparse_attn_kmeans_noalloc(
        _ptr(x), B, H, N, d, C, iters, _ptr(centroids), _ptr(labels), _ptr(perm), _ptr(offsets),
        _ptr(err_flag), _stream(stream)))


def sparse_attn_wait_selftest(err_flag, rounds, waited, stream=None):
    _check(load_library().sparse_attn_wait_selftest(_ptr(err_flag), rounds, _ptr(waited),
                                                    _stream(stream)))


def sparse_attn_permute_rows(src, perm, B, H, N, row_bytes, gather, dst, stream=None):
    _check(load_library().sparse_attn_permute_rows(
        _ptr(src), _ptr(perm), B, H, N, row_bytes, int(gather), _ptr(dst), _stream(stream)))


def sparse_attn_structured_mask(B, H, Nq, Nk, block, frame_tokens, n_frames, window, n_anchors,
                                period, step, q_frame0, kv_idx, kv_cnt, cap, stream=None):
    _check(load_library().sparse_attn_structured_mask(
        B, H, Nq, Nk, block, frame_tokens, n_frames, window, n_anchors, period, step, q_frame0,
        _ptr(kv_idx), _ptr(kv_cnt), cap, _stream(stream)))


def sparse_attn_structured_mask_adaptive(B, H, Nq, Nk, block, frame_tokens, n_frames, window,
                                         n_anchors, period, step, q_frame0, budget, kv_idx, kv_cnt,
                                         cap, stream=None):
    _check(load_library().sparse_attn_structured_mask_adaptive(
        B, H, Nq, Nk, block, frame_tokens, n_frames, window, n_anchors, period, step, q_frame0,
        budget, _ptr(kv_idx), _ptr(kv_cnt), cap, _stream(stream)))


def sparse_attn_forward(q, k, v16, kbar16, vsum16, M, kv_idx, kv_cnt, cap, B, H, Nq, Nk, d, block,
                        order, scale, out, out_dtype, err_flag=None, stream=None):
    _check(load_library().sparse_attn_forward(
        _ptr(q), _ptr(k), _ptr(v16), _ptr(kbar16), _ptr(vsum16), _ptr(M), _ptr(kv_idx),
        _ptr(kv_cnt), cap, B, H, Nq, Nk, d, block, order, scale, _ptr(out), out_dtype,
        _ptr(err_flag), _stream(stream)))


def sparse_attn_forward_split(q, k, v16, kbar16, vsum16, M, kv_idx, kv_cnt, cap, B, H, Nq, Nk, d,
                              block, order, scale, splits, work, out, out_dtype, err_flag=None,
                              stream=None):
    _check(load_library().sparse_attn_forward_split(
        _ptr(q), _ptr(k), _ptr(v16), _ptr(kbar16), _ptr(vsum16), _ptr(M), _ptr(kv_idx),
        _ptr(kv_cnt), cap, B, H, Nq, Nk, d, block, order, scale, splits, _ptr(work), _ptr(out),
        out_dtype, _ptr(err_flag), _stream(stream)))


def sparse_attn_forward_work_bytes(B, H, Nq, d, splits) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().sparse_attn_forward_work_bytes(B, H, Nq, d, splits, ctypes.byref(out)))
    return int(out.value)


def sparse_attn_forward_split_plan(B, H, Nq, Nk, d, block, sms=0):
    """(splits, work bytes) the library picks for this shape on ``sms`` SMs (0: the
    current device's count)."""
    n = _I(0)
    b = ctypes.c_size_t(0)
    _check(load_library().sparse_attn_forward_split_plan(B, H, Nq, Nk, d, block, sms,
                                                         ctypes.byref(n), ctypes.byref(b)))
    return int(n.value), int(b.value)


def sparse_attn_last_error() -> str:
    return load_library().sparse_attn_last_error().decode()
