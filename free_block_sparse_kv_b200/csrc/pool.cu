// Block pooling: query centroids, KV centroids, value sums and the per-block
// first-order matrices M_j = sum_r (k_r - kbar_j) v_r^T.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2 (Implémentation Matérielle: the pre-computation of block
// centroids and value sums; Algorithme Central: kbar_j and sum_n v_{j,n}) with the
// first-order term kept per block, and "SVG-EAR" §2 B (query centroids).
//
// The pass is HBM-bound: it reads Q, K, V once and writes M and an fp16 copy of V
// once. One persistent CTA per SM walks a static share of the work units (a KV block,
// or two query blocks, of some head) through a ring of shared-memory stages, with
// warp-specialised roles so that the loads, the products, the epilogue and the stores of
// different units overlap. Every reduction runs on the tensor cores, against a constant
// tile of ones in shared memory (bf16 products with 1 are exact, sums in fp32):
//   warp 8     TMA loads of each unit's K and V tiles (or its two Q tiles) into the next
//              free stage (128-byte swizzle; rows past the end of the tensor read as 0);
//   warp 10    one thread issues the unit's tcgen05.mma products into TMEM:
//                K^T V  (order 1; A = the K tile read M-major, i.e. transposed; B = V),
//                K^T 1  (every column = sum_r k_r: the centroid times n_j),
//                1^T V  (every row = sum_r v_r = S_j),
//              or Q^T 1 for each query block of a query unit;
//   warps 4-7  the epilogue, thread = TMEM lane a: kbar_a, S, qbar_a and the tables;
//              (order 1) M row a = (K^T V)[a] - kbar_a S, staged as fp16 in the stage's K
//              tile in the layout of a TMA store;
//   warps 0-3  convert the V tile to fp16 in place once the products have read it;
//   warp 9     TMA stores of the unit's fp16 V copy and M_j; hands the stage back to the
//              loader once the stores have read it.
// Every fp16 value written is checked: one that does not fit (|x| >= 65520 rounds to
// infinity) sets SA_FLAG_RANGE in err_flag.
#include "../../include/sparse_attn.h"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace sa {
namespace pl {

constexpr int kGroup = 128;                 // threads of the conversion group and of the epilogue
constexpr int kThreads = 2 * kGroup + 96;   // + load, store and MMA warps
constexpr uint32_t kWaitLimit = 1u << 18;   // ~0.3 s: far above any legitimate wait
constexpr int kWhere = 14;                  // err_flag bit of a pool wait that gave up

template <int D, int BLK, int ORDER>
struct Geom {
  static constexpr int SUB = D / 64;                 // 64-column sub-tiles per row
  static constexpr int CPR = D / 8;                  // 16-byte chunks per row
  static constexpr int RPP = kGroup / CPR;           // rows covered per pass of the group
  static constexpr int TILE = SUB * BLK * 128;       // one K, V or Q tile
  static constexpr int MBYTES = D * D * 2;           // one M_j in fp16
  // M is staged in the stage's K tile when it fits there, else in a slot of its own
  static constexpr bool MSEP = ORDER == 1 && MBYTES > TILE;
  static constexpr int STAGE = 2 * TILE + (MSEP ? MBYTES : 0);
  static constexpr int ONES = 128 * 128;             // 128 rows x 64 bf16 ones (16 KB)
  static constexpr int NS = ((212 * 1024 - ONES) / STAGE) < 4 ? ((212 * 1024 - ONES) / STAGE) : 4;
  static constexpr int OFF_ONES = NS * STAGE;
  static constexpr int OFF_CTL = OFF_ONES + ONES;
  static constexpr int SMEM = OFF_CTL + 512 + 1024;  // + alignment slack
  // TMEM columns: K^T V at [0, D), K^T 1 (or the first query block's Q^T 1) at
  // [C2, C2 + 64), 1^T V (or the second query block's Q^T 1) at [C3, C3 + D)
  static constexpr int C2 = D, C3 = 2 * D, TCOLS = 4 * D;
  static_assert(NS >= 2, "pool stages");
  static_assert(kGroup % CPR == 0, "pool geometry");
};

struct Ctl {
  uint64_t full[4], empty[4], vconv[4], mready[4], mdone[4];
  uint64_t tfull, tfree;
  uint32_t tmem;
  int abort;
};

struct Params {
  CUtensorMap tmK, tmV, tmQ, tmV16, tmM;
  float *qbar, *kbar_t, *vsum;
  uint16_t *kbar16, *vsum16;
  int32_t* err_flag;
  int Nq, Nk, nqb, nkb, j0, nkv, nq2, BH;
  long long units;
};

struct Unit {
  bool kv;
  int bh, idx;  // KV: block index j (j0 .. nkb-1); query: the pair of blocks 2 idx, 2 idx + 1
};

// Work units: every KV block of every head, then every pair of query blocks.
SA_DEVI Unit unit_of(const Params& p, long long u) {
  const long long nkv_all = (long long)p.BH * p.nkv;
  if (u < nkv_all) return Unit{true, (int)(u / p.nkv), p.j0 + (int)(u % p.nkv)};
  u -= nkv_all;
  return Unit{false, (int)(u / p.nq2), (int)(u % p.nq2)};
}

// Byte offset of 16-byte chunk c (0 .. d/8-1) of row r in a tile of `rows` rows:
// 64-column sub-tiles of rows x 128 B, chunks XOR-swizzled by the row within 8-row
// groups (the 128-byte swizzle of TMA and the tensor cores, 1024-byte-aligned base).
SA_DEVI uint32_t swz128(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// True when an fp16 pair holds an infinity (a value that did not fit).
SA_DEVI bool f16x2_inf(uint32_t h) {
  return (h & 0x7fffu) == 0x7c00u || (h & 0x7fff0000u) == 0x7c000000u;
}

// Barrier of the conversion group (named barrier 1) that also ORs a predicate over it.
SA_DEVI bool group_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"((uint32_t)pred), "n"(kGroup) : "memory");
  return r != 0;
}

template <int D, int BLK, int ORDER>
__global__ void __launch_bounds__(kThreads, 1) pool_kernel(const __grid_constant__ Params p) {
  using G = Geom<D, BLK, ORDER>;
  constexpr int NS = G::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  Ctl& c = *reinterpret_cast<Ctl*>(gbase + G::OFF_CTL);
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) {
    c.abort = 0;
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(bar(c.full[s]), 1);
      tc::mbar_init(bar(c.empty[s]), 1);
      tc::mbar_init(bar(c.vconv[s]), 4);
      tc::mbar_init(bar(c.mready[s]), 4);
      tc::mbar_init(bar(c.mdone[s]), 1);
    }
    tc::mbar_init(bar(c.tfull), 1);
    tc::mbar_init(bar(c.tfree), 4);
    tc::fence_mbar_init();
  }
  if (warp < 4) {
    // the ones tile: 128 rows of 64 bf16 ones (any swizzle of it is the same)
    uint4* o = reinterpret_cast<uint4*>(gbase + G::OFF_ONES);
    for (int x = tid; x < G::ONES / 16; x += kGroup) o[x] = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
    tc::fence_proxy_async();  // read by the tensor cores
  }
  if (warp == 9) {
    tc::tmem_alloc(smem_u32(&c.tmem), G::TCOLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = c.tmem;
  tc::Waiter wt{&c.abort, p.err_flag, kWaitLimit};
  const long long stride = gridDim.x;

  if (warp == 8) {
    // ================================ loads ================================
    if (lane == 0) {
      int n = 0;
      for (long long u = blockIdx.x; u < p.units; u += stride, ++n) {
        const int s = n % NS;
        if (n >= NS && !wt.fast(bar(c.empty[s]), ((n / NS) - 1) & 1, kWhere)) break;
        const Unit un = unit_of(p, u);
        const uint32_t st = base + s * G::STAGE, fb = bar(c.full[s]);
        if (un.kv) {
          tc::mbar_arrive_expect_tx(fb, 2 * G::TILE);
          for (int x = 0; x < G::SUB; ++x) {
            tc::tma_load_3d(st + x * BLK * 128, &p.tmK, fb, 64 * x, un.idx * BLK, un.bh);
            tc::tma_load_3d(st + G::TILE + x * BLK * 128, &p.tmV, fb, 64 * x, un.idx * BLK, un.bh);
          }
        } else {
          const int two = 2 * un.idx + 1 < p.nqb ? 2 : 1;
          tc::mbar_arrive_expect_tx(fb, two * G::TILE);
          for (int h = 0; h < two; ++h)
            for (int x = 0; x < G::SUB; ++x)
              tc::tma_load_3d(st + h * G::TILE + x * BLK * 128, &p.tmQ, fb, 64 * x,
                              (2 * un.idx + h) * BLK, un.bh);
        }
      }
      // every load issued lands before the CTA exits
      for (int m = n - NS > 0 ? n - NS : 0; m < n; ++m)
        tc::wait_drain(bar(c.full[m % NS]), (m / NS) & 1, kWaitLimit);
    }
  } else if (warp == 9) {
    // ================================ stores ===============================
    if (lane == 0) {
      int n = 0;
      for (long long u = blockIdx.x; u < p.units; u += stride, ++n) {
        const int s = n % NS;
        const uint32_t par = (n / NS) & 1;
        if (!wt.fast(bar(c.vconv[s]), par, kWhere)) break;
        const Unit un = unit_of(p, u);
        if (un.kv) {
          if (ORDER == 1 && !wt.fast(bar(c.mready[s]), par, kWhere)) break;
          const uint32_t st = base + s * G::STAGE;
          const uint32_t mst = G::MSEP ? st + 2 * G::TILE : st;
          for (int x = 0; x < G::SUB; ++x)
            tc::tma_store_3d(&p.tmV16, st + G::TILE + x * BLK * 128, 64 * x, un.idx * BLK, un.bh);
          if (ORDER == 1)
            for (int x = 0; x < G::SUB; ++x)
              tc::tma_store_3d(&p.tmM, mst + x * D * 128, 64 * x, 0, un.bh * p.nkb + un.idx);
          tc::bulk_commit();
          tc::bulk_wait_read();  // the stage may be refilled once the stores have read it
        }
        tc::mbar_arrive(bar(c.empty[s]));
      }
      tc::bulk_wait_all();
    }
  } else if (warp == 10) {
    // ================================ products ================================
    if (lane == 0) {
      const uint32_t ones = base + G::OFF_ONES;
      // A = a K or Q tile read M-major (rows = dims, K = tokens); B = a V tile or the
      // ones tile read N-major (rows = tokens); or A = the ones tile read K-major.
      constexpr uint32_t I_KV = tc::idesc_f16_mn(1, 1, 1, 1, D, 128);
      constexpr uint32_t I_K1 = tc::idesc_f16_mn(1, 1, 1, 1, 64, 128);
      constexpr uint32_t I_1V = tc::idesc_f16_mn(1, 1, 0, 1, D, 128);
      const uint64_t d1 = tc::sdesc(ones, BLK * 128, 1024);   // ones as N-major B (N = 64)
      const uint64_t da = tc::sdesc(ones, 16, 1024);          // ones as K-major A
      int n = 0;
      for (long long u = blockIdx.x; u < p.units; u += stride, ++n) {
        const int s = n % NS;
        if (!wt.fast(bar(c.full[s]), (n / NS) & 1, kWhere)) break;
        if (n >= 1 && !wt.fast(bar(c.tfree), (n - 1) & 1, kWhere)) break;
        tc::fence_after_sync();
        const Unit un = unit_of(p, u);
        const uint32_t st = base + s * G::STAGE;
        // K-steps of 16 tokens: 2048 bytes down an M- or N-major tile; 32 bytes along a
        // K-major row of the ones tile (whose 64 columns repeat for tokens 64 .. 127)
        auto tok = [](int kk) { return (uint64_t)((kk * 2048) >> 4); };
        auto row = [](int kk) { return (uint64_t)(((kk % 4) * 32) >> 4); };
        if (un.kv) {
          const uint64_t ak = tc::sdesc(st, BLK * 128, 1024);
          const uint64_t bv = tc::sdesc(st + G::TILE, BLK * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < BLK / 16; ++kk) {
            if (ORDER == 1) tc::mma_ss(tmem, ak + tok(kk), bv + tok(kk), I_KV, kk > 0);
            tc::mma_ss(tmem + G::C2, ak + tok(kk), d1 + tok(kk), I_K1, kk > 0);
            tc::mma_ss(tmem + G::C3, da + row(kk), bv + tok(kk), I_1V, kk > 0);
          }
        } else {
          const int two = 2 * un.idx + 1 < p.nqb ? 2 : 1;
          for (int h = 0; h < two; ++h) {
            const uint64_t aq = tc::sdesc(st + h * G::TILE, BLK * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < BLK / 16; ++kk)
              tc::mma_ss(tmem + (h ? G::C3 : G::C2), aq + tok(kk), d1 + tok(kk), I_K1, kk > 0);
          }
        }
        tc::mma_commit(bar(c.tfull));
        tc::mma_commit(bar(c.mdone[s]));
      }
      // products still in flight after an abort complete before TMEM is released
      if (n >= 1) tc::wait_drain(bar(c.tfull), (n - 1) & 1, kWaitLimit);
    }
  } else if (warp < 4) {
    // ============================ fp16 copy of V ============================
    constexpr int CPR = G::CPR, RPP = G::RPP;
    const int ch = tid % CPR, r0 = tid / CPR;
    bool bad = false;  // an fp16 value written by this thread overflowed
    // A wait every thread of the group ends alike: thread 0 waits on the barrier, and the
    // group barrier that ORs the outcome also orders what thread 0 observed (completed
    // products) before the other threads' accesses.
    auto group_wait = [&](uint32_t b, uint32_t par) {
      const bool got = tid == 0 ? wt.fast(b, par, kWhere) : !*wt.abort;
      return !group_sync_or(!got);
    };
    int n = 0;
    for (long long u = blockIdx.x; u < p.units; u += stride, ++n) {
      const int s = n % NS;
      // the unit's products have read the stage (per-stage barrier: no later product can
      // complete on it before this group releases the stage)
      if (!group_wait(bar(c.mdone[s]), (n / NS) & 1)) break;
      const Unit un = unit_of(p, u);
      if (un.kv) {
        uint8_t* sv = gbase + s * G::STAGE + G::TILE;
        for (int r = r0; r < BLK; r += RPP) {
          uint4* x = reinterpret_cast<uint4*>(sv + swz128(r, ch, BLK));
          const uint4 v = *x;
          const uint4 h = make_uint4(bf16x2_to_f16x2(v.x), bf16x2_to_f16x2(v.y),
                                     bf16x2_to_f16x2(v.z), bf16x2_to_f16x2(v.w));
          bad |= f16x2_inf(h.x) | f16x2_inf(h.y) | f16x2_inf(h.z) | f16x2_inf(h.w);
          *x = h;
        }
        // the converted tile is read by a TMA store (async proxy) after the arrival
        tc::fence_proxy_async();
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(c.vconv[s]));
    }
    if (p.err_flag && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err_flag, SA_FLAG_RANGE);
  } else {
    // ================================ epilogue ================================
    const int q4 = warp - 4;          // TMEM lane quadrant of this warp
    const int a = 32 * q4 + lane;     // dimension (TMEM lane, row of M) of this thread
    const uint32_t lq = (uint32_t)(32 * q4) << 16;
    bool bad = false;
    int n = 0;
    for (long long u = blockIdx.x; u < p.units; u += stride, ++n) {
      const int s = n % NS;
      if (!__all_sync(0xffffffffu, wt.fast(bar(c.tfull), n & 1, kWhere))) break;
      tc::fence_after_sync();
      const Unit un = unit_of(p, u);
      if (!un.kv) {
        // ---- two query blocks: qbar_i = (Q^T 1)[a] / n_i ----
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * un.idx + h;
          if (i >= p.nqb) break;
          const float sum = __uint_as_float(tc::tmem_ld1(tmem + lq + (h ? G::C3 : G::C2)));
          tc::tmem_wait_ld();
          if (a < D) p.qbar[((size_t)un.bh * p.nqb + i) * D + a] = sum / (float)min(BLK, p.Nq - i * BLK);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar(c.tfree));
        continue;
      }
      // ---- KV block j ----
      const int j = un.idx;
      const int n_j = min(BLK, p.Nk - j * BLK);
      const float ksum = __uint_as_float(tc::tmem_ld1(tmem + lq + G::C2));
      tc::tmem_wait_ld();
      const float ka = ksum / (float)n_j;  // centroid, dimension a
      if (a < D) {
        p.kbar_t[((size_t)un.bh * D + a) * p.nkb + j] = ka;
        // bf16 hi/lo split: hi = rn(kbar), lo = rn(kbar - hi); plane 0 then plane 1
        const __nv_bfloat16 hi = __float2bfloat16_rn(ka);
        const __nv_bfloat16 lo = __float2bfloat16_rn(ka - __bfloat162float(hi));
        p.kbar16[((size_t)(2 * un.bh) * p.nkb + j) * D + a] = *reinterpret_cast<const uint16_t*>(&hi);
        p.kbar16[((size_t)(2 * un.bh + 1) * p.nkb + j) * D + a] = *reinterpret_cast<const uint16_t*>(&lo);
      }
      uint8_t* st = gbase + s * G::STAGE;
      uint8_t* mst = G::MSEP ? st + 2 * G::TILE : st;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        // S_c for c = c0 .. c0 + 31: every TMEM lane of 1^T V holds the whole S
        uint32_t sv[32];
        tc::tmem_ld32(tmem + lq + G::C3 + c0, sv);
        tc::tmem_wait_ld();
        if (c0 == 32 * q4) {
          // this warp writes S_c for its own 32 dimensions: lane l the entry c0 + l
          float sl = __uint_as_float(sv[0]);
#pragma unroll
          for (int e = 1; e < 32; ++e) sl = lane == e ? __uint_as_float(sv[e]) : sl;
          const size_t row = ((size_t)un.bh * p.nkb + j) * D + c0 + lane;
          p.vsum[row] = sl;
          __half hs = __float2half_rn(sl);
          const uint16_t hb = *reinterpret_cast<uint16_t*>(&hs);
          bad |= (hb & 0x7fffu) == 0x7c00u;
          p.vsum16[row] = hb;
        }
        if constexpr (ORDER == 1) {
          // M row a = (K^T V)[a] - kbar_a S, fp16, in the layout of the TMA store
          uint32_t x[32];
          tc::tmem_ld32(tmem + lq + c0, x);
          tc::tmem_wait_ld();
          if (a < D) {
            uint32_t h[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              h[e] = pack_f16(fmaf(-ka, __uint_as_float(sv[2 * e]), __uint_as_float(x[2 * e])),
                              fmaf(-ka, __uint_as_float(sv[2 * e + 1]), __uint_as_float(x[2 * e + 1])));
              bad |= f16x2_inf(h[e]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
              *reinterpret_cast<uint4*>(mst + swz128(a, c0 / 8 + e, D)) =
                  make_uint4(h[4 * e], h[4 * e + 1], h[4 * e + 2], h[4 * e + 3]);
          }
        }
      }
      // TMEM released for the next unit's products; the staged M is read by a TMA store
      tc::fence_before_sync();
      if (ORDER == 1) tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(bar(c.tfree));
        if (ORDER == 1) tc::mbar_arrive(bar(c.mready[s]));
      }
    }
    if (p.err_flag && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.err_flag, SA_FLAG_RANGE);
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 9) tc::tmem_dealloc(tmem, G::TCOLS);
}

int sm_count() {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

template <int D, int BLK, int ORDER>
static cudaError_t launch_t(const PoolArgs& a, cudaStream_t st) {
  using G = Geom<D, BLK, ORDER>;
  Params p{};
  const int BH = a.B * a.H;
  const int nkv = a.Nk > 0 ? a.nkb - a.j0 : 0;
  const int nq2 = a.q ? (a.nqb + 1) / 2 : 0;
  p.units = (long long)BH * (nkv + nq2);
  if (p.units == 0) return cudaSuccess;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  bool ok = true;
  if (nkv > 0) {
    ok = map3d(&p.tmK, BF, a.k, D, a.Nk, BH, BLK) && map3d(&p.tmV, BF, a.v, D, a.Nk, BH, BLK) &&
         map3d(&p.tmV16, HF, a.v16, D, a.Nk, BH, BLK);
    if (ORDER == 1) ok = ok && map3d(&p.tmM, HF, a.M, D, D, (uint64_t)BH * a.nkb, D);
  }
  if (nq2 > 0) ok = ok && map3d(&p.tmQ, BF, a.q, D, a.Nq, BH, BLK);
  if (!ok) return cudaErrorInvalidValue;
  p.qbar = a.qbar;
  p.kbar_t = a.kbar_t;
  p.vsum = a.vsum;
  p.kbar16 = a.kbar16;
  p.vsum16 = a.vsum16;
  p.err_flag = a.err_flag;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.nqb = a.nqb;
  p.nkb = a.nkb;
  p.j0 = a.j0;
  p.nkv = nkv;
  p.nq2 = nq2;
  p.BH = BH;
  auto kern = pool_kernel<D, BLK, ORDER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const long long sms = sm_count();
  const unsigned grid = (unsigned)(p.units < sms ? p.units : sms);
  kern<<<grid, kThreads, G::SMEM, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pl

cudaError_t launch_pool(const PoolArgs& p, cudaStream_t st) {
  // order 2 (global first-order term) needs the per-block matrices like order 1
  const int order = p.order == 2 ? 1 : p.order;
#define SA_POOL_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && order == O_) return pl::launch_t<D_, B_, O_>(p, st);
  SA_POOL_CASE(64, 64, 0) SA_POOL_CASE(64, 64, 1) SA_POOL_CASE(64, 128, 0) SA_POOL_CASE(64, 128, 1)
  SA_POOL_CASE(128, 64, 0) SA_POOL_CASE(128, 64, 1) SA_POOL_CASE(128, 128, 0) SA_POOL_CASE(128, 128, 1)
#undef SA_POOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
