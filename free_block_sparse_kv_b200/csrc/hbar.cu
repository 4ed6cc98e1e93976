// Global first-order statistic and per-block covariance norms.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2: Algorithme Central (the global first-order matrix Hbar, the mean
// of the per-block first-order matrices over all blocks, used for every skipped block
// in place of its own matrix) and Routage Sensible à la Covariance (the norm of
// H_j - Hbar that enters the selection score; taken here over the matrix entries).
//
// Both kernels read the fp16 table of the per-block matrices M_j = H_j that the pool
// writes. They are HBM-bound: the mean reads the table once; the norms read it once
// more, with Hbar served from L2.
#include "common.cuh"
#include "launch.h"

namespace sa {

constexpr int kHbarThreads = 256;

// Hbar = (1/nkb) sum_j M_j. Thread x of the head owns 8 consecutive entries.
template <int D>
__global__ void __launch_bounds__(kHbarThreads)
hbar_mean_kernel(const uint16_t* __restrict__ M, int nkb, float* __restrict__ hbar,
                 uint16_t* __restrict__ hbar16) {
  const int bh = blockIdx.y;
  const int x = blockIdx.x * kHbarThreads + threadIdx.x;  // 8-entry chunk of the d x d matrix
  if (x >= D * D / 8) return;
  const uint16_t* src = M + (size_t)bh * nkb * D * D + (size_t)x * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < nkb; ++j) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (size_t)j * D * D));
    const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 p = *reinterpret_cast<const __half2*>(&h[e]);
      acc[2 * e] += __low2float(p);
      acc[2 * e + 1] += __high2float(p);
    }
  }
  const float inv = 1.f / (float)nkb;
  float* dst = hbar + (size_t)bh * D * D + (size_t)x * 8;
  uint32_t packed[4];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] *= inv;
  reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
#pragma unroll
  for (int e = 0; e < 4; ++e) packed[e] = pack_f16(acc[2 * e], acc[2 * e + 1]);
  *reinterpret_cast<uint4*>(hbar16 + (size_t)bh * D * D + (size_t)x * 8) =
      make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

// cov_j = sqrt(sum over entries of (M_j - Hbar)^2); one CTA per block.
template <int D>
__global__ void __launch_bounds__(kHbarThreads)
cov_kernel(const uint16_t* __restrict__ M, const float* __restrict__ hbar, int nkb,
           float* __restrict__ cov) {
  __shared__ float wsum[kHbarThreads / 32];
  const int j = blockIdx.x, bh = blockIdx.y;
  const uint16_t* mj = M + ((size_t)bh * nkb + j) * D * D;
  const float* hb = hbar + (size_t)bh * D * D;
  float s = 0.f;
  for (int x = threadIdx.x; x < D * D / 8; x += kHbarThreads) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(mj + (size_t)x * 8));
    const float4 h0 = __ldg(reinterpret_cast<const float4*>(hb + (size_t)x * 8));
    const float4 h1 = __ldg(reinterpret_cast<const float4*>(hb + (size_t)x * 8 + 4));
    const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
    const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 p = *reinterpret_cast<const __half2*>(&h[e]);
      const float d0 = __low2float(p) - hv[2 * e], d1 = __high2float(p) - hv[2 * e + 1];
      s = fmaf(d0, d0, s);
      s = fmaf(d1, d1, s);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kHbarThreads / 32; ++w) t += wsum[w];
    cov[(size_t)bh * nkb + j] = sqrtf(t);
  }
}

template <int D>
static cudaError_t launch_hbar_t(const HbarArgs& a, cudaStream_t st) {
  const int bh = a.B * a.H;
  dim3 g1((D * D / 8 + kHbarThreads - 1) / kHbarThreads, bh);
  hbar_mean_kernel<D><<<g1, kHbarThreads, 0, st>>>(a.M, a.nkb, a.hbar, a.hbar16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || a.cov == nullptr) return e;
  dim3 g2(a.nkb, bh);
  cov_kernel<D><<<g2, kHbarThreads, 0, st>>>(a.M, a.hbar, a.nkb, a.cov);
  return cudaGetLastError();
}

cudaError_t launch_hbar(const HbarArgs& a, cudaStream_t st) {
  if (a.d == 64) return launch_hbar_t<64>(a, st);
  if (a.d == 128) return launch_hbar_t<128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
