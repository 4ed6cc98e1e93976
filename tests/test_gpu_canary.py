"""Out-of-bounds write checks (in place of a sanitizer): every output buffer of every entry
point sits between two guard regions filled with a canary pattern, and the guards must be
intact after the call. Small and ragged shapes (N <= 512) are used, where index arithmetic
near the ends matters most; their results are also checked against the oracle."""
import numpy as np
import pytest
import torch

from free_block_sparse_kv_b200 import attention as A
from free_block_sparse_kv_b200 import sparse_attn as C
from free_block_sparse_kv_b200 import workloads as W
from oracle import block_sparse_attention as O
from oracle import cluster_layout as K

pytestmark = pytest.mark.gpu

PAD = 4096  # guard bytes on each side (a multiple of 256, so the middle stays aligned)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    C.load_library()


class Guarded:
    """A tensor of the given shape and dtype inside a byte buffer with canary guards."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((PAD + n + PAD,), 0xA5, dtype=torch.uint8, device="cuda")
        self.t = self.raw[PAD:PAD + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        g = torch.cat([self.raw[:PAD], self.raw[-PAD:]])
        return bool((g == 0xA5).all())


def _bits(shape, seed):
    rng = np.random.default_rng(seed)
    return W.bf16_round(rng.standard_normal(shape).astype(np.float32))[1]


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("N,d,block,order", [(300, 64, 64, 1), (129, 128, 128, 0),
                                             (512, 128, 64, 2), (77, 64, 128, 1)])
def test_pool_route_forward_stay_in_bounds(N, d, block, order):
    B, H = 1, 2
    qb, kb, vb = (_bits((B, H, N, d), 70 + s) for s in range(3))
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    p = A.Problem(B, H, N, N, d, block, order)
    f32, h16 = torch.float32, torch.float16
    g = dict(qbar=Guarded((B, H, p.nqb, d), f32), kbar_t=Guarded((B, H, d, p.nkb), f32),
             vsum=Guarded((B, H, p.nkb, d), f32), kbar16=Guarded((B, H, 2, p.nkb, d), torch.bfloat16),
             vsum16=Guarded((B, H, p.nkb, d), h16), v16=Guarded((B, H, N, d), h16),
             M=Guarded((B, H, p.nkb, d, d), h16) if order >= 1 else None,
             hbar=Guarded((B, H, d, d), f32) if order == 2 else None,
             hbar16=Guarded((B, H, d, d), h16) if order == 2 else None,
             cov=Guarded((B, H, p.nkb), f32) if order == 2 else None)
    t = A.Tables(**{name: (x.t if x is not None else None) for name, x in g.items()})
    A.pool(q, k, v, p, t)
    keep = -(-p.nkb // 3)
    idx = Guarded((B, H, p.nqb, keep), torch.int32, torch.full((B, H, p.nqb, keep), -7, dtype=torch.int32))
    cnt = Guarded((B, H, p.nqb), torch.int32)
    mode = "topk_cov" if order == 2 else "topk"
    A.route(p, t, idx.t, cnt.t, mode, rho=(1, 3))
    out = Guarded((B, H, N, d), f32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.forward(q, k, v, p, t, idx.t, cnt.t, out.t, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for name, x in list(g.items()) + [("kv_idx", idx), ("kv_cnt", cnt), ("out", out)]:
        if x is not None:
            assert x.intact(), name
    scale = 1 / np.sqrt(d)
    for h in range(H):
        qh, kh, vh = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        kept = O.route_head(qh, kh, block, mode, scale, keep=keep, v=vh)[0]
        want = O.forward_head(qh, kh, vh, kept, block, order, scale)
        got = out.t[0, h].cpu().numpy()
        assert np.abs(got - want).max() <= 1e-2


@pytest.mark.parametrize("Nq,d,splits,out_dtype", [(77, 64, 2, torch.float32),
                                                    (300, 128, 3, torch.bfloat16),
                                                    (129, 128, 5, torch.float32)])
def test_split_forward_stays_in_bounds(Nq, d, splits, out_dtype):
    """Partial results and the merge write inside their buffers (scratch sized exactly as
    the library states); 9,000 keys at block 64 give three runs of 64 blocks."""
    B, H, Nk, block, order = 1, 2, 9000, 64, 1
    qb, kb, vb = _bits((B, H, Nq, d), 90), _bits((B, H, Nk, d), 91), _bits((B, H, Nk, d), 92)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    p = A.Problem(B, H, Nq, Nk, d, block, order)
    t = A.allocate_tables(p, "cuda")
    A.pool(q, k, v, p, t)
    keep = -(-p.nkb // 6)
    idx = torch.empty(B, H, p.nqb, keep, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, H, p.nqb, dtype=torch.int32, device="cuda")
    A.route(p, t, idx, cnt, "topk", rho=(1, 6))
    work = Guarded((C.sparse_attn_forward_work_bytes(B, H, Nq, d, splits) // 4,), torch.float32)
    out = Guarded((B, H, Nq, d), out_dtype)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    A.forward(q, k, v, p, t, idx, cnt, out.t, err_flag=flag, splits=splits, work=work.t)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert work.intact() and out.intact()
    scale = 1 / np.sqrt(d)
    for h in range(H):
        qh, kh, vh = (W.bits_to_f32(x[0, h]) for x in (qb, kb, vb))
        kept = O.route_head(qh, kh, block, "topk", scale, keep=keep)[0]
        want = O.forward_head(qh, kh, vh, kept, block, order, scale)
        got = out.t[0, h].float().cpu().numpy()
        assert np.abs(got - want).max() <= 1e-2


def test_ear_kmeans_permute_stay_in_bounds():
    B, H, N, d, block = 1, 2, 333, 128, 64
    qb, kb, vb = (_bits((B, H, N, d), 80 + s) for s in range(3))
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    p = A.Problem(B, H, N, N, d, block, 0)
    t = A.allocate_tables(p, "cuda", ear=True)
    A.pool(q, k, v, p, t)
    sc = Guarded((B, H, p.nqb, p.nkb), torch.float32)
    C.sparse_attn_ear_scores(t.qbar, k, v, B, H, p.nqb, N, d, block, 1 / np.sqrt(d), sc.t)
    Cn, iters = 7, 2
    _, s_cw, s_iw = C.sparse_attn_kmeans_sizes(B, H, N, d, Cn)
    cent = Guarded((B, H, Cn, d), torch.float64)
    cw = Guarded((s_cw,), torch.uint8)
    iw = Guarded((s_iw // 4,), torch.int32)
    lab, perm = Guarded((B, H, N), torch.int32), Guarded((B, H, N), torch.int32)
    offs = Guarded((B, H, Cn + 1), torch.int32)
    C.sparse_attn_kmeans(k, B, H, N, d, Cn, iters, cent.t, cw.t, iw.t, lab.t, perm.t, offs.t)
    kp = Guarded((B, H, N, d), torch.bfloat16)
    A.permute_rows(k, perm.t, kp.t, gather=True)
    back = Guarded((B, H, N, d), torch.bfloat16)
    A.permute_rows(kp.t, perm.t, back.t, gather=False)
    torch.cuda.synchronize()
    for name, x in (("scores", sc), ("centroids", cent), ("cwork", cw), ("iwork", iw),
                    ("labels", lab), ("perm", perm), ("offsets", offs), ("gathered", kp),
                    ("scattered", back)):
        assert x.intact(), name
    assert torch.equal(back.t, k)
    kh = W.bits_to_f32(kb[0, 0])
    want_lab, _ = K.kmeans(kh, Cn, iters)
    assert np.array_equal(lab.t[0, 0].cpu().numpy(), want_lab)
