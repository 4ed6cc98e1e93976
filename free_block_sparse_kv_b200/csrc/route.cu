// Routing from pooled scores, and the structured (window + rotating anchor) mask.
//
// Routing follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient
// Diffusion Transformers" §2 (top-k choice of the critical blocks S_i) with the
// pooled proxies of "SVG-EAR" §2 B (query-block centroids stand in for the
// block's queries). The structured mask follows "LVSA: Training-Free Sparse
// Attention for Long Video Diffusion" §2 (A(t) = G u W(t), anchors shifted by
// s mod T_per).
//
// Route kernel: one CTA of 8 warps per (batch*head, 8 query blocks).
//   1. Scores s_ij = scale * qbar_i . kbar_j in fp32: thread j streams column j of
//      the dim-major centroid table (coalesced), the 8 qbar rows are broadcast from
//      shared memory.
//   2. One warp per query block selects. Each block gets the 48-bit key
//      (order-preserving bits of s) << 16 | (0xFFFF - j), so that larger keys come
//      first in the order (s descending, j ascending) and all keys differ. A
//      most-significant-bit-first search finds the threshold key T:
//        top-k:  the largest T with #{key >= T} >= k   (the k-th key)
//        mass:   the largest T with sum_{key >= T} e^(s - max) >= tau * Z
//      and the kept set is {key >= T}, written in ascending j with ballots.
#include "common.cuh"
#include "launch.h"

namespace sa {

constexpr int kRouteRows = 8;      // query blocks per CTA (one warp each)
constexpr int kRouteThreads = 256;

SA_DEVI uint64_t route_key(float s, int j) {
  return ((uint64_t)float_key(s) << 16) | (uint64_t)(0xFFFF - j);
}

template <int D>
__global__ void __launch_bounds__(kRouteThreads)
route_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar_t, int nqb, int nkb,
             int mode, int keep, float tau, float scale, int32_t* __restrict__ kv_idx,
             int32_t* __restrict__ kv_cnt, int cap) {
  extern __shared__ __align__(16) float rsm[];
  float* qs = rsm;                         // [D][kRouteRows]
  float* sc = rsm + D * kRouteRows;        // [kRouteRows][nkb] scores
  float* ex = sc + kRouteRows * nkb;       // [kRouteRows][nkb] e^(s - max) (mass mode)
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * kRouteRows;
  const int rows = min(kRouteRows, nqb - i0);

  for (int x = tid; x < D * kRouteRows; x += kRouteThreads) {
    const int r = x % kRouteRows, c = x / kRouteRows;
    qs[x] = (r < rows) ? qbar[((size_t)bh * nqb + i0 + r) * D + c] : 0.f;
  }
  __syncthreads();

  const float* kt = kbar_t + (size_t)bh * D * nkb;
  for (int j = tid; j < nkb; j += kRouteThreads) {
    float acc[kRouteRows];
#pragma unroll
    for (int r = 0; r < kRouteRows; ++r) acc[r] = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float kv = kt[(size_t)c * nkb + j];
      const float4 qa = *reinterpret_cast<const float4*>(qs + c * kRouteRows);
      const float4 qb = *reinterpret_cast<const float4*>(qs + c * kRouteRows + 4);
      acc[0] = fmaf(qa.x, kv, acc[0]);
      acc[1] = fmaf(qa.y, kv, acc[1]);
      acc[2] = fmaf(qa.z, kv, acc[2]);
      acc[3] = fmaf(qa.w, kv, acc[3]);
      acc[4] = fmaf(qb.x, kv, acc[4]);
      acc[5] = fmaf(qb.y, kv, acc[5]);
      acc[6] = fmaf(qb.z, kv, acc[6]);
      acc[7] = fmaf(qb.w, kv, acc[7]);
    }
#pragma unroll
    for (int r = 0; r < kRouteRows; ++r) sc[r * nkb + j] = scale * acc[r];
  }
  __syncthreads();

  const int warp = tid / 32, lane = tid % 32;
  if (warp >= rows) return;
  const float* s = sc + warp * nkb;
  const size_t row = (size_t)bh * nqb + i0 + warp;

  uint64_t prefix = 0;
  if (mode == 0) {
    for (int bit = 47; bit >= 0; --bit) {
      const uint64_t cand = prefix | (1ull << bit);
      int cnt = 0;
      for (int j = lane; j < nkb; j += 32) cnt += route_key(s[j], j) >= cand;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= keep) prefix = cand;
    }
  } else {
    float mx = -INFINITY;
    for (int j = lane; j < nkb; j += 32) mx = fmaxf(mx, s[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float* e = ex + warp * nkb;
    float z = 0.f;
    for (int j = lane; j < nkb; j += 32) {
      const float w = expf(s[j] - mx);
      e[j] = w;
      z += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float goal = tau * z;
    __syncwarp();
    for (int bit = 47; bit >= 0; --bit) {
      const uint64_t cand = prefix | (1ull << bit);
      float m = 0.f;
      for (int j = lane; j < nkb; j += 32)
        if (route_key(s[j], j) >= cand) m += e[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
      if (m >= goal) prefix = cand;
    }
  }

  int32_t* out = kv_idx + row * cap;
  int off = 0;
  for (int base = 0; base < nkb; base += 32) {
    const int j = base + lane;
    const bool in = j < nkb && route_key(s[j], j) >= prefix;
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (in) {
      const int pos = off + __popc(bal & ((1u << lane) - 1u));
      if (pos < cap) out[pos] = j;
    }
    off += __popc(bal);
  }
  if (lane == 0) kv_cnt[row] = min(off, cap);
}

template <int D>
static cudaError_t launch_route_t(const RouteArgs& p, cudaStream_t st) {
  const size_t smem = (size_t)(D * kRouteRows + 2 * kRouteRows * p.nkb) * sizeof(float);
  auto kern = route_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nqb + kRouteRows - 1) / kRouteRows, p.B * p.H);
  kern<<<grid, kRouteThreads, smem, st>>>(p.qbar, p.kbar_t, p.nqb, p.nkb, p.mode, p.keep, p.tau,
                                          p.scale, p.kv_idx, p.kv_cnt, p.cap);
  return cudaGetLastError();
}

cudaError_t launch_route(const RouteArgs& p, cudaStream_t st) {
  if (p.d == 64) return launch_route_t<64>(p, st);
  if (p.d == 128) return launch_route_t<128>(p, st);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Structured mask: one thread per (batch*head, query block). The query block's
// frames form one interval [f_lo, f_hi]; the union of their windows is
// [f_lo - window, f_hi + window]. Key block j (frames [g_lo, g_hi]) is kept when
// that interval meets [g_lo, g_hi] or when an anchor frame lies in [g_lo, g_hi].
// ---------------------------------------------------------------------------
__global__ void structured_mask_kernel(MaskArgs p) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)p.B * p.H * p.nqb) return;
  const int i = (int)(tid % p.nqb);
  const int ft = p.frame_tokens;
  const int qs = i * p.block, qe = min(p.Nq, qs + p.block) - 1;
  const int f_lo = p.q_frame0 + qs / ft, f_hi = p.q_frame0 + qe / ft;
  const int w_lo = f_lo - p.window, w_hi = f_hi + p.window;
  const int base = p.step % p.period;
  int32_t* out = p.kv_idx + tid * p.cap;
  int cnt = 0;
  for (int j = 0; j < p.nkb; ++j) {
    const int ks = j * p.block, ke = min(p.Nk, ks + p.block) - 1;
    const int g_lo = ks / ft, g_hi = ke / ft;
    bool keep = max(g_lo, w_lo) <= min(g_hi, w_hi);
    if (!keep) {
      // smallest anchor frame >= g_lo
      const int m = g_lo <= base ? 0 : (g_lo - base + p.period - 1) / p.period;
      const int a = base + m * p.period;
      keep = m < p.n_anchors && a <= g_hi && a < p.n_frames;
    }
    if (keep) {
      if (cnt < p.cap) out[cnt] = j;
      ++cnt;
    }
  }
  p.kv_cnt[tid] = min(cnt, p.cap);
}

cudaError_t launch_structured_mask(const MaskArgs& p, cudaStream_t st) {
  const long long n = (long long)p.B * p.H * p.nqb;
  const int threads = 128;
  structured_mask_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace sa
