// Block pooling: query centroids, KV centroids, value sums and the per-block
// first-order matrices M_j = sum_r (k_r - kbar_j) v_r^T.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2 (Implémentation Matérielle: the pre-computation of block
// centroids and value sums; Algorithme Central: kbar_j and sum_n v_{j,n}) with the
// first-order term kept per block, and "SVG-EAR" §2 B (query centroids).
//
// One CTA per block. KV CTAs stage the block's K and V tiles in shared memory
// with 16-byte cp.async (rows past the end zero-filled), reduce the column sums,
// and for order 1 compute K^T V on the tensor cores (mma.sync m16n8k16, fp32
// accumulate), subtract kbar S^T in fp32, and store M as fp16 through a
// swizzled shared-memory stage so that the global stores are 16-byte coalesced.
// It also writes an fp16 copy of V, the value operand of the forward's exact
// products. The pass is HBM-bound: it reads Q, K, V once and writes M and V16 once.
#include "common.cuh"
#include "launch.h"

namespace sa {

constexpr int kPoolThreads = 256;

template <int D, int BLK, int ORDER>
__global__ void __launch_bounds__(kPoolThreads, 2)
pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
            const uint16_t* __restrict__ v, int Nq, int Nk, int nqb, int nkb,
            float* __restrict__ qbar, float* __restrict__ kbar_t, float* __restrict__ vsum,
            uint16_t* __restrict__ kbar16, uint16_t* __restrict__ vsum16,
            uint16_t* __restrict__ M, uint16_t* __restrict__ v16) {
  constexpr int ROWB = D * 2;             // bytes per bf16 row
  constexpr int CPR = D / 8;              // 16-byte chunks per row
  constexpr int RPP = kPoolThreads / CPR; // rows covered per pass
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sk = smem;                     // BLK x D bf16, swizzled
  uint8_t* sv = smem + BLK * ROWB;        // BLK x D bf16, swizzled
  float* red = reinterpret_cast<float*>(smem + 2 * BLK * ROWB);  // [2][RPP][D]
  float* ks = red + 2 * RPP * D;          // [D] key column sums -> centroid
  float* vs = ks + D;                     // [D] value sums

  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  const int ch = tid % CPR;
  const int r0 = tid / CPR;

  if (blk >= nkb) {
    // ---- query block: qbar_i = mean of its rows ----
    const int i = blk - nkb;
    const int start = i * BLK;
    const int n = min(BLK, Nq - start);
    const uint16_t* src = q + ((size_t)bh * Nq + start) * D;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = r0; r < n; r += RPP) {
      uint4 x = *reinterpret_cast<const uint4*>(src + (size_t)r * D + ch * 8);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += bf16_lo(w[e]);
        acc[2 * e + 1] += bf16_hi(w[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r0 * D + ch * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
      for (int p = 0; p < RPP; ++p) s += red[p * D + tid];
      qbar[((size_t)bh * nqb + i) * D + tid] = s / (float)n;
    }
    return;
  }

  // ---- KV block j ----
  const int j = blk;
  const int start = j * BLK;
  const int n = min(BLK, Nk - start);
  const uint16_t* kg = k + ((size_t)bh * Nk + start) * D;
  const uint16_t* vg = v + ((size_t)bh * Nk + start) * D;
  const uint32_t skb = smem_u32(sk), svb = smem_u32(sv);
  for (int r = r0; r < BLK; r += RPP) {
    const bool ok = r < n;
    const size_t off = ok ? (size_t)r * D + ch * 8 : 0;
    cp_async16(skb + swz(r, ch, ROWB), kg + off, ok ? 16 : 0);
    cp_async16(svb + swz(r, ch, ROWB), vg + off, ok ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  {
    float ak[8] = {0, 0, 0, 0, 0, 0, 0, 0}, av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint16_t* v16g = v16 + ((size_t)bh * Nk + start) * D;
    for (int r = r0; r < n; r += RPP) {
      const uint4 xk = *reinterpret_cast<const uint4*>(sk + swz(r, ch, ROWB));
      const uint4 xv = *reinterpret_cast<const uint4*>(sv + swz(r, ch, ROWB));
      const uint32_t wk[4] = {xk.x, xk.y, xk.z, xk.w}, wv[4] = {xv.x, xv.y, xv.z, xv.w};
      *reinterpret_cast<uint4*>(v16g + (size_t)r * D + ch * 8) =
          make_uint4(bf16x2_to_f16x2(xv.x), bf16x2_to_f16x2(xv.y), bf16x2_to_f16x2(xv.z),
                     bf16x2_to_f16x2(xv.w));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ak[2 * e] += bf16_lo(wk[e]);
        ak[2 * e + 1] += bf16_hi(wk[e]);
        av[2 * e] += bf16_lo(wv[e]);
        av[2 * e + 1] += bf16_hi(wv[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[r0 * D + ch * 8 + e] = ak[e];
      red[(RPP + r0) * D + ch * 8 + e] = av[e];
    }
  }
  __syncthreads();
  if (tid < 2 * D) {
    const int c = tid % D;
    const int which = tid / D;  // 0: keys, 1: values
    float s = 0.f;
    for (int p = 0; p < RPP; ++p) s += red[(which * RPP + p) * D + c];
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
    __syncthreads();
    // M = K^T V - kbar S^T. Warps: 4 along a (key dim) x 2 along c (value dim).
    constexpr int WA = D / 4, WC = D / 2;
    constexpr int MT = WA / 16, NT = WC / 8;
    const int warp = tid / 32, lane = tid % 32;
    const int a0 = (warp / 2) * WA, c0 = (warp % 2) * WC;
    float acc[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < BLK / 16; ++kk) {
      uint32_t af[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int r = kk * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int col = a0 + mt * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(skb + swz(r, col / 8, ROWB), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = c0 + np * 16 + ((lane >> 4) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(svb + swz(r, col / 8, ROWB), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_bf16(acc[mt][2 * np], af[mt], b0, b1);
          mma_bf16(acc[mt][2 * np + 1], af[mt], b2, b3);
        }
      }
    }
    __syncthreads();  // every warp is done reading sk: reuse it as the M stage
    const int g = lane / 4, t = lane % 4;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int a = a0 + mt * 16 + g + hf * 8;
          const int c = c0 + nt * 8 + 2 * t;
          const float x0 = acc[mt][nt][2 * hf] - ks[a] * vs[c];
          const float x1 = acc[mt][nt][2 * hf + 1] - ks[a] * vs[c + 1];
          *reinterpret_cast<uint32_t*>(sk + swz(a, c / 8, ROWB) + (c % 8) * 2) = pack_f16(x0, x1);
        }
    __syncthreads();
    uint16_t* mg = M + ((size_t)bh * nkb + j) * D * D;
    for (int a = r0; a < D; a += RPP)
      *reinterpret_cast<uint4*>(mg + (size_t)a * D + ch * 8) =
          *reinterpret_cast<const uint4*>(sk + swz(a, ch, ROWB));
  }
}

template <int D, int BLK, int ORDER>
static cudaError_t launch_pool_t(const PoolArgs& p, cudaStream_t st) {
  constexpr int ROWB = D * 2;
  constexpr int RPP = kPoolThreads / (D / 8);
  const size_t smem = 2 * (size_t)BLK * ROWB + (2 * RPP * D + 2 * D) * sizeof(float);
  auto kern = pool_kernel<D, BLK, ORDER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int nq_blocks = p.q ? p.nqb : 0;
  dim3 grid(p.nkb + nq_blocks, p.B * p.H);
  kern<<<grid, kPoolThreads, smem, st>>>(p.q, p.k, p.v, p.Nq, p.Nk, p.nqb, p.nkb, p.qbar,
                                         p.kbar_t, p.vsum, p.kbar16, p.vsum16, p.M, p.v16);
  return cudaGetLastError();
}

cudaError_t launch_pool(const PoolArgs& p, cudaStream_t st) {
#define SA_POOL_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && p.order == O_) return launch_pool_t<D_, B_, O_>(p, st);
  SA_POOL_CASE(64, 64, 0) SA_POOL_CASE(64, 64, 1) SA_POOL_CASE(64, 128, 0) SA_POOL_CASE(64, 128, 1)
  SA_POOL_CASE(128, 64, 0) SA_POOL_CASE(128, 64, 1) SA_POOL_CASE(128, 128, 0) SA_POOL_CASE(128, 128, 1)
#undef SA_POOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
