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
//   warps 0-7  two groups of four warps, one thread per centroid row in each; group g
//              takes the blocks n = g, g+2, ... of the run: logits from TMEM, the weight
//              differences as bf16 hi + lo back into TMEM, then ||X||^2 and the score;
//   warp 8     TMA producer: K tiles (three stages) and V tiles (two), bf16 as given;
//   warps 9-10 MMA issuers, one thread each, warp 9 + g for group g's blocks:
//              S = (Qhi + Qlo) K^T, then X = (Phi + Plo) V. One thread issuing every
//              product could not keep the tensor cores busy: issuing one costs about as
//              long as the tensor cores take to run it at these shapes.
// The centroid tile is split into two bf16 pieces (16 significant bits) so that the
// logit differences s_r - s_c, which carry the error, keep about 16 bits; the weight
// differences are split into two bf16 pieces (truncation, about 16 bits; a bf16 split
// needs integer masks and byte permutes only, where fp16 needs conversions that share
// the special-function unit with the exponentials). Group g owns TMEM
// logit buffer g (BLK columns) and X buffer g (D columns), so the two groups work on
// consecutive blocks at once while the tensor cores run the other group's products.
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace sa {
namespace ear {

constexpr int kThreads = 352;
constexpr int TQ = 128;                       // centroid rows per tile
constexpr uint32_t kWaitLimit = 1u << 18;     // try_wait rounds before giving up

template <int D, int BLK>
struct Geom {
  static constexpr int SUB = D / 64;          // 64-column sub-tiles of a row
  static constexpr int QPIECE = TQ * D * 2;   // one bf16 piece of the centroid tile
  static constexpr int KT = BLK * D * 2;      // a K tile or a V tile
  static constexpr int CTL = 512;             // barriers and words
  // three K stages where they fit beside the centroid pieces and two V stages
  static constexpr int NKS = 2 * QPIECE + 5 * KT + CTL + 1024 <= 232448 ? 3 : 2;
  static constexpr int OFF_Q = 0;             // [2 pieces][SUB][TQ rows x 128 B]
  static constexpr int OFF_K = 2 * QPIECE;    // [NKS stages][SUB][BLK rows x 128 B]
  static constexpr int OFF_V = OFF_K + NKS * KT;  // [2 stages][SUB][BLK rows x 128 B]
  static constexpr int OFF_CTL = OFF_V + 2 * KT;
  static constexpr int COL_S = 0;             // logits / weight differences: [2][BLK]
  static constexpr int COL_X = 2 * BLK;       // X: [2][D]
  static constexpr int NCOL = 2 * BLK + 2 * D;
  static constexpr int TCOLS = NCOL <= 256 ? 256 : 512;
  // Shared memory is sized so that the CTAs resident on one SM never ask for more than
  // the SM's 512 TMEM columns: one CTA per SM with 512 columns, at most two with 256.
  static constexpr int NEED = OFF_CTL + CTL + 1024;  // + alignment slack
  static constexpr int FLOOR = TCOLS == 512 ? 232448 / 2 + 1024 : 232448 / 3 + 1024;
  static constexpr int SMEM = NEED > FLOOR ? NEED : FLOOR;
  static_assert(SMEM <= 232448, "shared memory");
};

struct Ctl {
  uint64_t k_full[3], k_empty[3], v_full[2], v_empty[2];
  uint64_t s_full[2], x_full[2], x_free[2];
  uint64_t p_full[2][4];  // per group, per chunk of 32 keys: its weight differences are in TMEM
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
    for (int b = 0; b < 3; ++b) {
      tc::mbar_init(bar(c.k_full[b]), 1);
      tc::mbar_init(bar(c.k_empty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(c.v_full[b]), 1);
      tc::mbar_init(bar(c.v_empty[b]), 1);
      tc::mbar_init(bar(c.s_full[b]), 1);
      tc::mbar_init(bar(c.x_full[b]), 1);
      for (int q = 0; q < 4; ++q) tc::mbar_init(bar(c.p_full[b][q]), TQ);
      tc::mbar_init(bar(c.x_free[b]), TQ);
    }
    tc::mbar_init(bar(c.done), 2);
    c.abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(smem_u32(&c.tmem_base), G::TCOLS);
    tc::tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
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

  if (warp < 8) {
    // ============ rows: weight differences, then the error of each block ============
    const int g = warp / 4;               // group: blocks n = g, g + 2, ...
    const int row = tid & (TQ - 1);       // TMEM lane and centroid row of the tile
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_off + G::COL_S + BLK * g;
    const uint32_t x_col = tmem + lane_off + G::COL_X + D * g;
    const float sl2 = p.scale * kLog2e;  // logits in base 2
    // warp-uniform outcome of a wait, so that the warp's TMEM accesses stay converged
    auto uni = [](bool x) { return __all_sync(0xffffffffu, x); };
    // One block of the run. FULL: all BLK keys valid (every block but a partial last one),
    // so the per-key validity selects drop out.
    auto unit = [&](int n, int nv, auto full) __attribute__((always_inline)) {
      constexpr bool FULL = decltype(full)::value;
      auto valid = [&](int r) { return FULL || r < nv; };
      const int par = (n >> 1) & 1;
      if (!uni(wt.wait(bar(c.s_full[g]), par, 1))) return false;
      tc::fence_after_sync();
      // pass 1: largest logit and the logit sum over the valid keys, 64 keys at a time
      float mx[2] = {-INFINITY, -INFINITY};
      uint64_t sm2[2] = {0, 0};
#pragma unroll
      for (int h = 0; h < BLK / 64; ++h) {
        uint32_t sr[64];
        tc::tmem_ld32(s_col + 64 * h, sr);
        tc::tmem_ld32(s_col + 64 * h + 32, sr + 32);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const int r = 64 * h + e;
          float v[4];
#pragma unroll
          for (int f = 0; f < 4; ++f) v[f] = valid(r + f) ? __uint_as_float(sr[e + f]) : -INFINITY;
          mx[0] = tc::max3(mx[0], v[0], v[1]);
          mx[1] = tc::max3(mx[1], v[2], v[3]);
#pragma unroll
          for (int f = 0; f < 4; ++f) v[f] = valid(r + f) ? __uint_as_float(sr[e + f]) : 0.f;
          sm2[(e / 4) & 1] =
              tc::add2(sm2[(e / 4) & 1], tc::add2(tc::f2(v[0], v[1]), tc::f2(v[2], v[3])));
        }
      }
      const float ms = fmaxf(mx[0], mx[1]);  // largest logit (natural units / scale)
      float a0, a1, b0, b1;
      tc::f2_split(sm2[0], a0, a1);
      tc::f2_split(sm2[1], b0, b1);
      const float mean = ((a0 + a1) + (b0 + b1)) / (float)nv;
      const float m2 = ms * sl2;  // base-2 logit of the block's largest weight
      const float wc = tc::ex2((mean - ms) * sl2);
      const uint64_t sl2x2 = tc::f2(sl2, sl2), nm2x2 = tc::f2(-m2, -m2), nwc = tc::f2(-wc, -wc);
      // pass 2: weight differences d_r = 2^(u_r - m) - 2^(u_c - m) as bf16 hi + lo, hi the
      // top 16 bits of d_r and lo = d_r - hi (exact in fp32) rounded to bf16; chunk q
      // of 32 keys goes to columns [32q, 32q + 16) (hi) and [32q + 16, 32q + 32) (lo),
      // which only overwrites logits of the chunk itself
#pragma unroll 1
      for (int q = 0; q < BLK / 32; ++q) {
        uint32_t sr[32], hi[16], lo[16];
        tc::tmem_ld32(s_col + 32 * q, sr);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int r = 32 * q + 2 * e;
          float e0, e1;
          tc::f2_split(tc::fma2(tc::f2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                sl2x2, nm2x2), e0, e1);
          float d0, d1;
          tc::f2_split(tc::add2(tc::f2(tc::ex2(e0), tc::ex2(e1)), nwc), d0, d1);
          d0 = valid(r) ? d0 : 0.f;
          d1 = valid(r + 1) ? d1 : 0.f;
          const uint32_t u0 = __float_as_uint(d0) & 0xFFFF0000u;
          const uint32_t u1 = __float_as_uint(d1) & 0xFFFF0000u;
          float l0, l1;
          tc::f2_split(tc::add2(tc::f2(d0, d1), tc::f2(-__uint_as_float(u0), -__uint_as_float(u1))),
                       l0, l1);
          hi[e] = __byte_perm(u0, u1, 0x7632);  // (hi0, hi1) as two bf16, hi0 in the low half
          // lo rounded half away from zero: a carry out of the low 16 bits rounds the magnitude
          lo[e] = __byte_perm(__float_as_uint(l0) + 0x8000u, __float_as_uint(l1) + 0x8000u, 0x7632);
        }
        tc::tmem_st16(s_col + 32 * q, hi);
        tc::tmem_st16(s_col + 32 * q + 16, lo);
        // the chunk's value products can start while the next chunk is computed
        tc::tmem_wait_st();
        tc::fence_before_sync();
        tc::mbar_arrive(bar(c.p_full[g][q]));
      }

      // the block's error: ||X||^2 with X = sum_r d_r v_r
      if (!uni(wt.wait(bar(c.x_full[g]), par, 3))) return false;
      tc::fence_after_sync();
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t xr[64];
        tc::tmem_ld32(x_col + 64 * h, xr);
        tc::tmem_ld32(x_col + 64 * h + 32, xr + 32);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const uint64_t xv = tc::f2(__uint_as_float(xr[e]), __uint_as_float(xr[e + 1]));
          acc[(e / 2) & 3] = tc::fma2(xv, xv, acc[(e / 2) & 3]);
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(bar(c.x_free[g]));
      float t0, t1, t2, t3, t4, t5, t6, t7;
      tc::f2_split(acc[0], t0, t1);
      tc::f2_split(acc[1], t2, t3);
      tc::f2_split(acc[2], t4, t5);
      tc::f2_split(acc[3], t6, t7);
      const float ss = ((t0 + t1) + (t2 + t3)) + ((t4 + t5) + (t6 + t7));
      if (row < rows) {
        const float score = (__log2f(ss) + 2.f * m2) * 0.6931471805599453f - __logf((float)nv);
        p.scores[((size_t)bh * p.nqb + i0 + row) * p.nkb + j0 + n] = score;
      }
      return true;
    };
    for (int n = g; n < nj; n += 2) {
      const int nv = min(BLK, p.Nk - (j0 + n) * BLK);  // valid keys of the block
      const bool ok = nv == BLK ? unit(n, nv, std::true_type{}) : unit(n, nv, std::false_type{});
      if (!ok) break;
    }
  } else if (warp == 8) {
    // ======================== TMA producer ========================
    // Loads go out in the order the products need them: K0, K1, then V_n, K_{n+2}.
    if (lane == 0) {
      constexpr int NKS = G::NKS;
      uint32_t kused = 0, kpar = 0, vused = 0, vpar = 0;  // per stage: loaded, last parity
      auto load_k = [&](int n) __attribute__((always_inline)) {
        const int st = n % NKS, ph = (n / NKS) & 1;
        if (n >= NKS && !wt.wait(bar(c.k_empty[st]), ph ^ 1, 4)) return false;
        tc::mbar_arrive_expect_tx(bar(c.k_full[st]), G::KT);
        for (int x = 0; x < G::SUB; ++x)
          tc::tma_load_3d(base + G::OFF_K + st * G::KT + x * BLK * 128, &p.tmK, bar(c.k_full[st]),
                          64 * x, (j0 + n) * BLK, bh);
        kused |= 1u << st;
        kpar = (kpar & ~(1u << st)) | ((uint32_t)ph << st);
        return true;
      };
      auto load_v = [&](int n) __attribute__((always_inline)) {
        const int st = n & 1, ph = (n >> 1) & 1;
        if (n >= 2 && !wt.wait(bar(c.v_empty[st]), ph ^ 1, 5)) return false;
        tc::mbar_arrive_expect_tx(bar(c.v_full[st]), G::KT);
        for (int x = 0; x < G::SUB; ++x)
          tc::tma_load_3d(base + G::OFF_V + st * G::KT + x * BLK * 128, &p.tmV, bar(c.v_full[st]),
                          64 * x, (j0 + n) * BLK, bh);
        vused |= 1u << st;
        vpar = (vpar & ~(1u << st)) | ((uint32_t)ph << st);
        return true;
      };
      bool ok = load_k(0) && (nj < 2 || load_k(1));
      for (int n = 0; n < nj && ok; ++n) ok = load_v(n) && (n + 2 >= nj || load_k(n + 2));
      // Every load issued must land before the CTA exits.
      for (int st = 0; st < NKS; ++st)
        if ((kused >> st) & 1) tc::wait_drain(bar(c.k_full[st]), (kpar >> st) & 1, kWaitLimit);
      for (int st = 0; st < 2; ++st)
        if ((vused >> st) & 1) tc::wait_drain(bar(c.v_full[st]), (vpar >> st) & 1, kWaitLimit);
    }
  } else if (warp == 9 || warp == 10) {
    // ================ MMA issuers: warp 9 + g for the blocks of group g ================
    if (lane == 0) {
      constexpr int NKS = G::NKS;
      constexpr uint32_t I_S = tc::idesc_f16(1, 1, 0, BLK);
      constexpr uint32_t I_PV = tc::idesc_f16(1, 1, 1, D);
      const int g = warp - 9;
      const uint64_t dq = tc::sdesc(base + G::OFF_Q, 16, 1024);
      const uint32_t sd = tmem + G::COL_S + BLK * g, xd = tmem + G::COL_X + D * g;
      // logits of block n into this group's buffer
      auto issue_s = [&](int n) __attribute__((always_inline)) {
        const int st = n % NKS;
        if (!wt.wait(bar(c.k_full[st]), (n / NKS) & 1, 6)) return false;
        tc::fence_after_sync();
        const uint64_t dk = tc::sdesc(base + G::OFF_K + st * G::KT, 16, 1024);
        for (int pc = 0; pc < 2; ++pc) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = (pc * G::QPIECE + (kk / 4) * TQ * 128 + (kk % 4) * 32) >> 4;
            const uint32_t boff = ((kk / 4) * BLK * 128 + (kk % 4) * 32) >> 4;
            tc::mma_ss(sd, dq + aoff, dk + boff, I_S, (pc | kk) > 0);
          }
        }
        tc::mma_commit(bar(c.s_full[g]));
        tc::mma_commit(bar(c.k_empty[st]));
        return true;
      };
      bool ok = g >= nj || issue_s(g);
      for (int n = g; n < nj && ok; n += 2) {
        const int par = (n >> 1) & 1;
        ok = wt.wait(bar(c.v_full[g]), par, 8) && (n < 2 || wt.wait(bar(c.x_free[g]), par ^ 1, 9));
        if (!ok) break;
        const uint64_t dv = tc::sdesc(base + G::OFF_V + g * G::KT, BLK * 128, 1024);
        // chunk q of 32 keys as soon as its weight differences are written: hi at columns
        // [32q, 32q + 16), lo 16 further, 16 keys (8 columns) per product
        for (int q = 0; q < BLK / 32 && ok; ++q) {
          ok = wt.wait(bar(c.p_full[g][q]), par, 7);
          if (!ok) break;
          tc::fence_after_sync();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t dvk = dv + (((2 * q + h) * 2048) >> 4);
            tc::mma_ts(xd, sd + 32 * q + 8 * h, dvk, I_PV, (q | h) > 0);
            tc::mma_ts(xd, sd + 32 * q + 16 + 8 * h, dvk, I_PV, 1);
          }
        }
        if (!ok) break;
        tc::mma_commit(bar(c.x_full[g]));
        tc::mma_commit(bar(c.v_empty[g]));
        // the next logits of this buffer, behind the products that read its P
        if (n + 2 < nj) ok = issue_s(n + 2);
      }
      // Every product issued is complete before TMEM is released (both issuers commit).
      tc::mma_commit(bar(c.done));
      tc::wait_drain(bar(c.done), 0, kWaitLimit);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 9) {
    __syncwarp();
    tc::tmem_dealloc(tmem, G::TCOLS);
  }
}

// Key blocks per CTA: the run length that minimises waves x (run + prologue), with one
// CTA per SM and the prologue (centroid tile, TMEM, barriers) costed as three blocks.
int choose_run(uint64_t tiles, int nkb) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 1;
  int best = 32;
  uint64_t best_cost = ~0ull;
  for (int run = 16; run <= 128; ++run) {
    const uint64_t ctas = tiles * (uint64_t)((nkb + run - 1) / run);
    const uint64_t cost = ((ctas + sms - 1) / sms) * (uint64_t)(run + 3);
    if (cost < best_cost) {
      best_cost = cost;
      best = run;
    }
    if (run >= nkb) break;  // longer runs change nothing
  }
  return best;
}

template <int D, int BLK>
cudaError_t launch_t(const EarArgs& a, cudaStream_t st) {
  using G = Geom<D, BLK>;
  Params p;
  const uint64_t bh = (uint64_t)a.B * a.H;
  if (!map3d(&p.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, D, a.Nk, bh, BLK) ||
      !map3d(&p.tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.v, D, a.Nk, bh, BLK))
    return cudaErrorInvalidValue;
  p.qbar = a.qbar;
  p.scores = a.scores;
  p.err_flag = a.err_flag;
  p.Nk = a.Nk;
  p.nqb = a.nqb;
  p.nkb = a.nkb;
  p.scale = a.scale;
  p.ntq = (a.nqb + TQ - 1) / TQ;
  p.run = a.run > 0 ? a.run : choose_run((uint64_t)p.ntq * bh, a.nkb);
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
