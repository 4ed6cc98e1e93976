// Error-aware routing scores: the per-block error of the centroid approximation.
//
// Follows "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video Generation
// via Error-aware Routing" §2 B (a light probe estimates, per key block, the squared
// error between exact attention and its centroid approximation, with the query
// centroids standing in for the queries, and ranks blocks by that error per unit of
// cost) and §2 C (the estimate is computed in one streaming pass; no logit reaches
// HBM).
//
// For query centroid qbar_i (a row of the pooled query table) and key block j with
// n_j tokens:
//   s_r = scale qbar_i . k_r,  s_c = (1/n_j) sum_r s_r  (= scale qbar_i . kbar_j),
//   m = max_r s_r,             X = sum_r (exp(s_r - m) - exp(s_c - m)) v_r,
//   score_ij = ln(||X||^2 / n_j) + 2 m       (= ln(err_ij / n_j), err = -inf if 0).
//
// Kernel: one CTA per (batch*head, tile of 128 centroids, run of key blocks).
//   warps 0-3  one thread per centroid row: logits from TMEM, the weight differences
//              as fp16 hi + lo back into TMEM, then ||X||^2 from TMEM and the score;
//   warp 4     TMA producer: K tiles (bf16) and V tiles (fp16), two stages each;
//   warp 5     MMA issuer (one thread): S = (Qhi + Qlo) K^T, then X = (Phi + Plo) V.
// The centroid tile is split into two bf16 pieces (16 significant bits) so that the
// logit differences s_r - s_c, which carry the error, keep about 16 bits; the weight
// differences are split into two fp16 pieces for the same reason. TMEM holds two
// logit buffers (BLK columns) and two X buffers (D columns), so the logits of block
// n+1 are computed while the rows finish block n.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace sa {
namespace ear {

constexpr int kThreads = 192;
constexpr int TQ = 128;                       // centroid rows per tile
constexpr uint32_t kWaitLimit = 1u << 18;     // try_wait rounds before giving up

template <int D, int BLK>
struct Geom {
  static constexpr int SUB = D / 64;          // 64-column sub-tiles of a row
  static constexpr int QPIECE = TQ * D * 2;   // one bf16 piece of the centroid tile
  static constexpr int KT = BLK * D * 2;      // a K tile or a V tile
  static constexpr int OFF_Q = 0;             // [2 pieces][SUB][TQ rows x 128 B]
  static constexpr int OFF_K = 2 * QPIECE;    // [2 stages][SUB][BLK rows x 128 B]
  static constexpr int OFF_V = OFF_K + 2 * KT;
  static constexpr int OFF_CTL = OFF_V + 2 * KT;
  static constexpr int COL_S = 0;             // logits / weight differences: [2][BLK]
  static constexpr int COL_X = 2 * BLK;       // X: [2][D]
  static constexpr int NCOL = 2 * BLK + 2 * D;
  static constexpr int TCOLS = NCOL <= 256 ? 256 : 512;
  // Shared memory is sized so that the CTAs resident on one SM never ask for more than
  // the SM's 512 TMEM columns: one CTA per SM with 512 columns, at most two with 256.
  static constexpr int NEED = OFF_CTL + 256 + 1024;  // + alignment slack
  static constexpr int FLOOR = TCOLS == 512 ? 232448 / 2 + 1024 : 232448 / 3 + 1024;
  static constexpr int SMEM = NEED > FLOOR ? NEED : FLOOR;
  static_assert(SMEM <= 232448, "shared memory");
};

struct Ctl {
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], x_full[2], x_free[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  CUtensorMap tmK, tmV;
  const float* qbar;
  float* scores;
  int32_t* err_flag;
  int Nk, nqb, nkb, ntq, nch, run;
  float scale;
};

// Byte offset of 16-byte chunk c of row r in a tile of `rows` rows stored as 64-column
// sub-tiles (rows x 128 B each) with the 128-byte swizzle.
SA_DEVI uint32_t swz128(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1) ear_kernel(const __grid_constant__ Params p) {
  using G = Geom<D, BLK>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t base = smem_u32(smem);
  Ctl& c = *reinterpret_cast<Ctl*>(smem + G::OFF_CTL);
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // CTA -> (head, run of key blocks, centroid tile); the tiles of one run are adjacent
  // so that they read the same K and V tiles while those are in L2.
  const int cta = blockIdx.x;
  const int t = cta % p.ntq;
  const int ch = (cta / p.ntq) % p.nch;
  const int bh = cta / (p.ntq * p.nch);
  const int j0 = ch * p.run;
  const int nj = min(p.run, p.nkb - j0);
  const int i0 = t * TQ;
  const int rows = min(TQ, p.nqb - i0);

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(c.k_full[b]), 1);
      tc::mbar_init(bar(c.v_full[b]), 1);
      tc::mbar_init(bar(c.k_empty[b]), 1);
      tc::mbar_init(bar(c.v_empty[b]), 1);
      tc::mbar_init(bar(c.s_full[b]), 1);
      tc::mbar_init(bar(c.x_full[b]), 1);
      tc::mbar_init(bar(c.p_full[b]), TQ);
      tc::mbar_init(bar(c.x_free[b]), TQ);
    }
    tc::mbar_init(bar(c.done), 1);
    c.abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(smem_u32(&c.tmem_base), G::TCOLS);
    tc::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tc::prefetch_tmap(&p.tmK);
    tc::prefetch_tmap(&p.tmV);
  }
  // The centroid tile as two bf16 pieces, hi = rn(x) and lo = rn(x - hi), in the
  // swizzled K-major layout the tensor cores read. Rows past the last block are zero.
  {
    constexpr int CPR = D / 8;  // 16-byte chunks (8 elements) per row
    const float* src = p.qbar + ((size_t)bh * p.nqb + i0) * D;
    for (int x = tid; x < TQ * CPR; x += kThreads) {
      const int r = x / CPR, ch8 = x % CPR;
      float v[8];
      if (r < rows) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(src + (size_t)r * D + ch8 * 8));
        const float4 b = __ldg(reinterpret_cast<const float4*>(src + (size_t)r * D + ch8 * 8 + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = 0.f;
      }
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hi[e] = pack_bf16(v[2 * e], v[2 * e + 1]);
        lo[e] = pack_bf16(v[2 * e] - bf16_lo(hi[e]), v[2 * e + 1] - bf16_hi(hi[e]));
      }
      const uint32_t off = swz128(r, ch8, TQ);
      *reinterpret_cast<uint4*>(smem + G::OFF_Q + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + G::OFF_Q + G::QPIECE + off) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    tc::fence_proxy_async();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  tc::Waiter wt{&c.abort, p.err_flag, kWaitLimit};

  if (warp < 4) {
    // ============ rows: weight differences, then the error of each block ============
    const int row = tid;  // TMEM lane and centroid row of the tile
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float sl2 = p.scale * kLog2e;  // logits in base 2
    float m_prev = 0.f;
    int nv_prev = 1;
    // warp-uniform outcome of a wait, so that the warp's TMEM accesses stay converged
    auto uni = [](bool x) { return __all_sync(0xffffffffu, x); };
    auto x_phase = [&](int n, float m2, int nv) __attribute__((always_inline)) {
      const int b = n & 1;
      if (!uni(wt.wait(bar(c.x_full[b]), (n >> 1) & 1, 3))) return false;
      tc::fence_after_sync();
      float ss = 0.f;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t xr[32];
        tc::tmem_ld32(tmem + lane_off + G::COL_X + D * b + 32 * q, xr);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float xv = __uint_as_float(xr[e]);
          ss = fmaf(xv, xv, ss);
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(bar(c.x_free[b]));
      if (row < rows) {
        const float score = (log2f(ss) + 2.f * m2) * 0.6931471805599453f - logf((float)nv);
        p.scores[((size_t)bh * p.nqb + i0 + row) * p.nkb + j0 + n] = score;
      }
      return true;
    };
    bool ok = true;
    for (int n = 0; n < nj && ok; ++n) {
      const int b = n & 1;
      const int nv = min(BLK, p.Nk - (j0 + n) * BLK);  // valid keys of the block
      ok = uni(wt.wait(bar(c.s_full[b]), (n >> 1) & 1, 1));
      if (!ok) break;
      tc::fence_after_sync();
      float u[BLK];
#pragma unroll
      for (int q = 0; q < BLK / 32; ++q)
        tc::tmem_ld32(tmem + lane_off + G::COL_S + BLK * b + 32 * q,
                      reinterpret_cast<uint32_t*>(u + 32 * q));
      tc::tmem_wait_ld();
      float m2 = -INFINITY;
#pragma unroll
      for (int r = 0; r < BLK; ++r) {
        u[r] *= sl2;
        if (r < nv) m2 = fmaxf(m2, u[r]);
      }
      float sum = 0.f;  // sum of (u_r - m): the centroid logit relative to the maximum
#pragma unroll
      for (int r = 0; r < BLK; ++r)
        if (r < nv) sum += u[r] - m2;
      const float wc = tc::ex2(sum / (float)nv);
#pragma unroll
      for (int q = 0; q < BLK / 32; ++q) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int r = 32 * q + 2 * e;
          const float d0 = r < nv ? tc::ex2(u[r] - m2) - wc : 0.f;
          const float d1 = r + 1 < nv ? tc::ex2(u[r + 1] - m2) - wc : 0.f;
          hi[e] = pack_f16(d0, d1);
          const __half2 h = *reinterpret_cast<const __half2*>(&hi[e]);
          lo[e] = pack_f16(d0 - __low2float(h), d1 - __high2float(h));
        }
        tc::tmem_st16(tmem + lane_off + G::COL_S + BLK * b + 16 * q, hi);
        tc::tmem_st16(tmem + lane_off + G::COL_S + BLK * b + BLK / 2 + 16 * q, lo);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(bar(c.p_full[b]));
      if (n > 0) ok = x_phase(n - 1, m_prev, nv_prev);
      m_prev = m2;
      nv_prev = nv;
    }
    if (ok && nj > 0) x_phase(nj - 1, m_prev, nv_prev);
  } else if (warp == 4) {
    // ======================== TMA producer ========================
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int n = 0; n < nj && ok; ++n) {
        const int b = n & 1, j = j0 + n;
        if (n >= 2) ok = wt.wait(bar(c.k_empty[b]), ((n >> 1) - 1) & 1, 4);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar(c.k_full[b]), G::KT);
        for (int x = 0; x < G::SUB; ++x)
          tc::tma_load_3d(base + G::OFF_K + b * G::KT + x * BLK * 128, &p.tmK, bar(c.k_full[b]),
                          64 * x, j * BLK, bh);
        if (n >= 2) ok = wt.wait(bar(c.v_empty[b]), ((n >> 1) - 1) & 1, 5);
        if (!ok) {
          issued = 2 * n + 1;
          break;
        }
        tc::mbar_arrive_expect_tx(bar(c.v_full[b]), G::KT);
        for (int x = 0; x < G::SUB; ++x)
          tc::tma_load_3d(base + G::OFF_V + b * G::KT + x * BLK * 128, &p.tmV, bar(c.v_full[b]),
                          64 * x, j * BLK, bh);
        issued = 2 * n + 2;
      }
      // Every load issued must land before the CTA exits: wait for the last two of each.
      for (int h = max(0, issued - 4); h < issued; ++h) {
        const int n = h / 2, b = n & 1;
        tc::wait_drain(bar(h % 2 ? c.v_full[b] : c.k_full[b]), (n >> 1) & 1, kWaitLimit);
      }
    }
  } else {
    // ======================== MMA issuer ========================
    if (lane == 0) {
      constexpr uint32_t I_S = tc::idesc_f16(1, 1, 0, BLK);
      constexpr uint32_t I_PV = tc::idesc_f16(0, 0, 1, D);
      const uint64_t dq = tc::sdesc(base + G::OFF_Q, 16, 1024);
      auto issue_s = [&](int n) __attribute__((always_inline)) {
        const int b = n & 1;
        if (!wt.wait(bar(c.k_full[b]), (n >> 1) & 1, 6)) return false;
        tc::fence_after_sync();
        const uint64_t dk = tc::sdesc(base + G::OFF_K + b * G::KT, 16, 1024);
        for (int pc = 0; pc < 2; ++pc) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = (pc * G::QPIECE + (kk / 4) * TQ * 128 + (kk % 4) * 32) >> 4;
            const uint32_t boff = ((kk / 4) * BLK * 128 + (kk % 4) * 32) >> 4;
            tc::mma_ss(tmem + G::COL_S + BLK * b, dq + aoff, dk + boff, I_S, (pc | kk) > 0);
          }
        }
        tc::mma_commit(bar(c.s_full[b]));
        tc::mma_commit(bar(c.k_empty[b]));
        return true;
      };
      bool ok = nj > 0 ? issue_s(0) : true;
      for (int n = 0; n < nj && ok; ++n) {
        const int b = n & 1;
        if (n + 1 < nj) ok = issue_s(n + 1);
        if (!ok) break;
        ok = wt.wait(bar(c.p_full[b]), (n >> 1) & 1, 7) &&
             wt.wait(bar(c.v_full[b]), (n >> 1) & 1, 8) &&
             (n < 2 || wt.wait(bar(c.x_free[b]), ((n >> 1) - 1) & 1, 9));
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t dv = tc::sdesc(base + G::OFF_V + b * G::KT, BLK * 128, 1024);
        const uint32_t pa = tmem + G::COL_S + BLK * b, xd = tmem + G::COL_X + D * b;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk)
          tc::mma_ts(xd, pa + kk * 8, dv + ((kk * 2048) >> 4), I_PV, kk > 0);
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk)
          tc::mma_ts(xd, pa + BLK / 2 + kk * 8, dv + ((kk * 2048) >> 4), I_PV, 1);
        tc::mma_commit(bar(c.x_full[b]));
        tc::mma_commit(bar(c.v_empty[b]));
      }
      // Every product issued is complete before TMEM is released.
      tc::mma_commit(bar(c.done));
      tc::wait_drain(bar(c.done), 0, kWaitLimit);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 5) {
    __syncwarp();
    tc::tmem_dealloc(tmem, G::TCOLS);
  }
}

template <int D, int BLK>
cudaError_t launch_t(const EarArgs& a, cudaStream_t st) {
  using G = Geom<D, BLK>;
  Params p;
  const uint64_t bh = (uint64_t)a.B * a.H;
  if (!map3d(&p.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, D, a.Nk, bh, BLK) ||
      !map3d(&p.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.v16, D, a.Nk, bh, BLK))
    return cudaErrorInvalidValue;
  p.qbar = a.qbar;
  p.scores = a.scores;
  p.err_flag = a.err_flag;
  p.Nk = a.Nk;
  p.nqb = a.nqb;
  p.nkb = a.nkb;
  p.scale = a.scale;
  p.ntq = (a.nqb + TQ - 1) / TQ;
  p.run = a.run > 0 ? a.run : 32;
  p.nch = (a.nkb + p.run - 1) / p.run;
  const uint64_t ctas = (uint64_t)p.ntq * p.nch * bh;
  if (ctas == 0) return cudaSuccess;
  if (ctas > 0x7fffffffull) return cudaErrorInvalidValue;
  auto kern = ear_kernel<D, BLK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)ctas, kThreads, G::SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace ear

cudaError_t launch_ear(const EarArgs& a, cudaStream_t st) {
  if (a.d == 64 && a.block == 64) return ear::launch_t<64, 64>(a, st);
  if (a.d == 64 && a.block == 128) return ear::launch_t<64, 128>(a, st);
  if (a.d == 128 && a.block == 64) return ear::launch_t<128, 64>(a, st);
  if (a.d == 128 && a.block == 128) return ear::launch_t<128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
