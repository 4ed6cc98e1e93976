// Block pooling: query centroids, KV centroids, value sums and the per-block
// first-order matrices M_j = sum_r (k_r - kbar_j) v_r^T.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2 (Implémentation Matérielle: the pre-computation of block
// centroids and value sums; Algorithme Central: kbar_j and sum_n v_{j,n}) with the
// first-order term kept per block, and "SVG-EAR" §2 B (query centroids).
//
// One CTA of 256 threads per block, three CTAs per SM (73 KB of shared memory, 128 TMEM
// columns and at most 85 registers each), so that the loads of one CTA overlap the
// reductions and stores of the others. A KV CTA stages the block's K and V tiles in
// shared memory with 16-byte cp.async in the 128-byte-swizzled layout of the tensor
// cores (64-column sub-tiles, rows past the end zero-filled), reduces the column sums
// (warp shuffles, then one shared row per warp), writes an fp16 copy of V (the value
// operand of the forward's exact products), and for order 1 computes K^T V with
// tcgen05.mma (A = the K tile read M-major, i.e. transposed; B = V; fp32 accumulator in
// TMEM), then subtracts kbar S^T in fp32 and stores M as fp16 rows. The pass is
// HBM-bound: it reads Q, K, V once and writes M and V16 once.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace sa {

constexpr int kPoolThreads = 256;
constexpr int kPoolWarps = kPoolThreads / 32;

template <int D, int BLK>
struct PoolGeom {
  static constexpr int SUB = D / 64;                 // 64-column sub-tiles per row
  static constexpr int CPR = D / 8;                  // 16-byte chunks per row
  static constexpr int RPP = kPoolThreads / CPR;     // rows covered per pass
  static constexpr int TILE = SUB * BLK * 128;       // one K, V or Q tile
  static constexpr int OFF_RED = 2 * TILE;           // [2][warps][D] partial column sums
  static constexpr int OFF_KS = OFF_RED + 2 * kPoolWarps * D * 4;  // [D] centroid, [D] value sum
  static constexpr int OFF_CTL = OFF_KS + 2 * D * 4;  // mbarrier, TMEM address
  static constexpr int SMEM = OFF_CTL + 64 + 1024;   // + alignment slack
  static constexpr int TCOLS = D < 32 ? 32 : D;      // TMEM allocation (power of two >= 32)
  static_assert(kPoolThreads % CPR == 0, "pool geometry");
};

// Byte offset of 16-byte chunk c (0 .. d/8-1) of row r in a tile of `rows` rows:
// 64-column sub-tiles of rows x 128 B, chunks XOR-swizzled by the row within 8-row
// groups (the tensor cores' 128-byte swizzle on a 1024-byte-aligned base).
SA_DEVI uint32_t swz128(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D, int BLK, int ORDER>
__global__ void __launch_bounds__(kPoolThreads, 3)
pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
            const uint16_t* __restrict__ v, int Nq, int Nk, int nqb, int nkb, int j0,
            float* __restrict__ qbar, float* __restrict__ kbar_t, float* __restrict__ vsum,
            uint16_t* __restrict__ kbar16, uint16_t* __restrict__ vsum16,
            uint16_t* __restrict__ M, uint16_t* __restrict__ v16) {
  using G = PoolGeom<D, BLK>;
  constexpr int CPR = G::CPR, RPP = G::RPP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sk = smem;                                 // K (or Q) tile
  uint8_t* sv = smem + G::TILE;                       // V tile
  float* red = reinterpret_cast<float*>(smem + G::OFF_RED);
  float* ks = reinterpret_cast<float*>(smem + G::OFF_KS);
  float* vs = ks + D;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + G::OFF_CTL);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + G::OFF_CTL + 8);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  const int ch = tid % CPR;
  const int r0 = tid / CPR;

  // Column sums of a staged tile: thread (r0, ch) adds rows r0, r0 + RPP, ... of its
  // 8 columns; lanes that share ch meet by shuffles, then one shared row per warp.
  auto colsum = [&](const uint8_t* tile, int n, float* out_rows) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = r0; r < n; r += RPP) {
      const uint4 x = *reinterpret_cast<const uint4*>(tile + swz128(r, ch, BLK));
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_lo(w[e]);
        acc[2 * e + 1] += bf16_hi(w[e]);
      }
    }
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (lane < CPR)
#pragma unroll
      for (int e = 0; e < 8; ++e) out_rows[warp * D + ch * 8 + e] = acc[e];
  };

  const int nkv = nkb - j0;  // KV blocks pooled by this launch: j0 .. nkb-1
  if (blk >= nkv) {
    // ---- query block: qbar_i = mean of its rows ----
    const int i = blk - nkv;
    const int start = i * BLK;
    const int n = min(BLK, Nq - start);
    const uint16_t* src = q + ((size_t)bh * Nq + start) * D;
    const uint32_t skb = smem_u32(sk);
    for (int r = r0; r < n; r += RPP) cp_async16(skb + swz128(r, ch, BLK), src + (size_t)r * D + ch * 8, 16);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    colsum(sk, n, red);
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
      for (int w = 0; w < kPoolWarps; ++w) s += red[w * D + tid];
      qbar[((size_t)bh * nqb + i) * D + tid] = s / (float)n;
    }
    return;
  }

  // ---- KV block j ----
  const int j = j0 + blk;
  const int start = j * BLK;
  const int n = min(BLK, Nk - start);
  const uint16_t* kg = k + ((size_t)bh * Nk + start) * D;
  const uint16_t* vg = v + ((size_t)bh * Nk + start) * D;
  const uint32_t skb = smem_u32(sk), svb = smem_u32(sv);
  for (int r = r0; r < BLK; r += RPP) {
    const bool ok = r < n;
    const size_t off = ok ? (size_t)r * D + ch * 8 : 0;
    cp_async16(skb + swz128(r, ch, BLK), kg + off, ok ? 16 : 0);
    cp_async16(svb + swz128(r, ch, BLK), vg + off, ok ? 16 : 0);
  }
  cp_async_commit();
  if constexpr (ORDER == 1) {
    if (warp == 0) {
      tc::tmem_alloc(smem_u32(tslot), G::TCOLS);
      tc::tmem_relinquish();
    }
    if (tid == 32) {
      tc::mbar_init(smem_u32(mbar), 1);
      tc::fence_mbar_init();
    }
  }
  cp_async_wait<0>();
  // the staged tiles are read by the tensor cores (async proxy) after this barrier
  tc::fence_proxy_async();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  uint32_t tmem = 0;
  if constexpr (ORDER == 1) {
    tmem = *tslot;
    if (tid == 0) {
      // K^T V: A = the K tile read M-major (rows a = key dims, K = tokens), B = the V
      // tile (tokens x value dims, N-major); 16 tokens per instruction. For d = 64 the
      // M = 128 instruction also computes 64 rows from the V tile that are not read.
      constexpr uint32_t idesc = tc::idesc_f16_mn(1, 1, 1, 1, D, 128);
      const uint64_t ad = tc::sdesc(skb, BLK * 128, 1024), bd = tc::sdesc(svb, BLK * 128, 1024);
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk)
        tc::mma_ss(tmem, ad + ((kk * 2048) >> 4), bd + ((kk * 2048) >> 4), idesc, kk > 0);
      tc::mma_commit(smem_u32(mbar));
    }
  }

  // fp16 copy of V and column sums (the tensor cores only read the tiles)
  {
    uint16_t* v16g = v16 + ((size_t)bh * Nk + start) * D;
    for (int r = r0; r < n; r += RPP) {
      const uint4 xv = *reinterpret_cast<const uint4*>(sv + swz128(r, ch, BLK));
      *reinterpret_cast<uint4*>(v16g + (size_t)r * D + ch * 8) =
          make_uint4(bf16x2_to_f16x2(xv.x), bf16x2_to_f16x2(xv.y), bf16x2_to_f16x2(xv.z),
                     bf16x2_to_f16x2(xv.w));
    }
  }
  colsum(sk, n, red);
  colsum(sv, n, red + kPoolWarps * D);
  __syncthreads();
  if (tid < 2 * D) {
    const int c = tid % D;
    const int which = tid / D;  // 0: keys, 1: values
    float s = 0.f;
    for (int w = 0; w < kPoolWarps; ++w) s += red[(which * kPoolWarps + w) * D + c];
    const size_t row = ((size_t)bh * nkb + j) * D + c;
    if (which == 0) {
      const float mean = s / (float)n;
      ks[c] = mean;
      kbar_t[((size_t)bh * D + c) * nkb + j] = mean;
      // bf16 hi/lo split: hi = rn(mean), lo = rn(mean - hi); plane 0 then plane 1
      const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
      const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
      kbar16[((size_t)(2 * bh) * nkb + j) * D + c] = *reinterpret_cast<const uint16_t*>(&hi);
      kbar16[((size_t)(2 * bh + 1) * nkb + j) * D + c] = *reinterpret_cast<const uint16_t*>(&lo);
    } else {
      vs[c] = s;
      vsum[row] = s;
      __half h = __float2half_rn(s);
      vsum16[row] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
  if constexpr (ORDER == 1) {
    __syncthreads();  // ks, vs visible
    // M = K^T V - kbar S^T. TMEM lane a holds row a; warps w and w + 4 take the two
    // column halves of lanes 32 (w % 4) ... A product that never completes (bounded
    // wait) leaves M unwritten rather than holding the CTA.
    const bool done = tc::wait_drain(smem_u32(mbar), 0, 1u << 20);
    tc::fence_after_sync();
    const int a = 32 * (warp & 3) + lane;
    constexpr int HC = D / 2;  // columns per thread
    constexpr int ROWB = D * 2;
    static_assert(D * ROWB <= 2 * G::TILE, "M stage");
    const float ka = a < D ? ks[a] : 0.f;
    // fp16 rows into the (consumed) K and V tiles, then coalesced 16-byte stores
#pragma unroll
    for (int cb = 0; cb < HC; cb += 32) {
      const int c0 = (warp >> 2) * HC + cb;
      uint32_t x[32];
      tc::tmem_ld32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + c0, x);
      tc::tmem_wait_ld();
      if (a < D) {
        uint32_t h[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          h[e] = pack_f16(__uint_as_float(x[2 * e]) - ka * vs[c0 + 2 * e],
                          __uint_as_float(x[2 * e + 1]) - ka * vs[c0 + 2 * e + 1]);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(sk + swz(a, c0 / 8 + e, ROWB)) =
              make_uint4(h[4 * e], h[4 * e + 1], h[4 * e + 2], h[4 * e + 3]);
      }
    }
    __syncthreads();
    if (done) {
      uint16_t* mg = M + ((size_t)bh * nkb + j) * D * D;
      for (int r = r0; r < D; r += RPP)
        *reinterpret_cast<uint4*>(mg + (size_t)r * D + ch * 8) =
            *reinterpret_cast<const uint4*>(sk + swz(r, ch, ROWB));
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, G::TCOLS);
  }
}

template <int D, int BLK, int ORDER>
static cudaError_t launch_pool_t(const PoolArgs& p, cudaStream_t st) {
  using G = PoolGeom<D, BLK>;
  auto kern = pool_kernel<D, BLK, ORDER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  const int nq_blocks = p.q ? p.nqb : 0;
  const int nkv = p.Nk > 0 ? p.nkb - p.j0 : 0;
  if (nkv + nq_blocks == 0) return cudaSuccess;
  dim3 grid(nkv + nq_blocks, p.B * p.H);
  kern<<<grid, kPoolThreads, G::SMEM, st>>>(p.q, p.k, p.v, p.Nq, p.Nk, p.nqb, p.nkb, p.j0, p.qbar,
                                            p.kbar_t, p.vsum, p.kbar16, p.vsum16, p.M, p.v16);
  return cudaGetLastError();
}

cudaError_t launch_pool(const PoolArgs& p, cudaStream_t st) {
  // order 2 (global first-order term) needs the per-block matrices like order 1
  const int order = p.order == 2 ? 1 : p.order;
#define SA_POOL_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && order == O_) return launch_pool_t<D_, B_, O_>(p, st);
  SA_POOL_CASE(64, 64, 0) SA_POOL_CASE(64, 64, 1) SA_POOL_CASE(64, 128, 0) SA_POOL_CASE(64, 128, 1)
  SA_POOL_CASE(128, 64, 0) SA_POOL_CASE(128, 64, 1) SA_POOL_CASE(128, 128, 0) SA_POOL_CASE(128, 128, 1)
#undef SA_POOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
