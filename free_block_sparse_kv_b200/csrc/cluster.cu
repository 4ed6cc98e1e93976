// k-means clustering of one tensor's rows per (batch, head) and the group-major token
// layout built from it.
//
// Follows "SVG-EAR: Parameter-Free Linear Compensation for Sparse Video Generation via
// Error-aware Routing" §2 A (query and key tokens grouped into semantic clusters by
// k-means before the sparse attention) and "Partition the Support, Reconstruct the
// Residual: Training-Free Sparse Attention for Video Generation and World Models" §2 C
// (tokens permuted into contiguous group-major layouts).
//
// Lloyd's iteration from the tokens at floor(m N / C): assign every token to its nearest
// centroid (ties to the lowest index), move every centroid to the mean of its members
// (one without members stays), and after the last update assign once more. The layout
// is the stable counting sort of the final labels.
//
// Kernels, per iteration:
//   assign   tcgen05: a tile of 128 tokens against tiles of 128 centroids,
//            S = X C_hi^T + X C_lo^T (the fp64 centroids as two bf16 pieces), score
//            ||c||^2 - 2 S in fp32; a token whose two best scores lie closer than the
//            error bound of that arithmetic goes on a list instead of being decided;
//   recheck  the listed tokens in fp64 against every centroid (one CTA each);
//   hist / scan / scatter   stable counting sort: one warp per chunk of 1024 tokens;
//   update   segments of at most 512 sorted members summed in fp64 by one CTA each, then
//            one CTA per cluster adds its segments (the sums of bf16 values are exact,
//            so the means are the correctly rounded fp64 means); the bf16 pieces and
//            fp32 squared norms the next assignment reads follow.
#include <cudaTypedefs.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace sa {
namespace km {

constexpr int TT = 128;                      // tokens per assignment tile
constexpr int TCN = 128;                     // centroids per tile
constexpr int kChunk = 1024;                 // tokens per sorting warp
constexpr int kSortWarps = 4;
constexpr int kSeg = 512;                    // members per centroid-update segment
constexpr uint32_t kWaitLimit = 1u << 18;

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------
// init and prep
// ---------------------------------------------------------------------------
__global__ void init_kernel(const uint16_t* __restrict__ x, int N, int d, int C,
                            double* __restrict__ cent) {
  const int m = blockIdx.x, bh = blockIdx.y;
  const long long r = (long long)m * N / C;
  const uint16_t* src = x + ((size_t)bh * N + r) * d;
  double* dst = cent + ((size_t)bh * C + m) * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    dst[i] = (double)__uint_as_float((uint32_t)src[i] << 16);
}

// The assignment's operands from the fp64 centroids: bf16 hi = rn(c), lo = rn(c - hi),
// and ||c||^2 in fp32; padding centroids (m >= C) get zero pieces and +inf. Also clears
// the head's list of undecided tokens.
__global__ void prep_kernel(const double* __restrict__ cent, int C, int Cpad, int d,
                            uint16_t* __restrict__ pieces, float* __restrict__ cnorm,
                            int32_t* __restrict__ amb_cnt) {
  const int m = blockIdx.x, bh = blockIdx.y;
  __shared__ double red[32];
  uint16_t* hi = pieces + (((size_t)bh * 2 + 0) * Cpad + m) * d;
  uint16_t* lo = pieces + (((size_t)bh * 2 + 1) * Cpad + m) * d;
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    if (m < C) {
      const double c = cent[((size_t)bh * C + m) * d + i];
      const float cf = (float)c;
      const __nv_bfloat16 h = __float2bfloat16_rn(cf);
      const float rest = (float)(c - (double)__bfloat162float(h));
      const __nv_bfloat16 l = __float2bfloat16_rn(rest);
      hi[i] = __bfloat16_as_ushort(h);
      lo[i] = __bfloat16_as_ushort(l);
      s += c * c;
    } else {
      hi[i] = 0;
      lo[i] = 0;
    }
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)blockDim.x / 32; ++w) t += red[w];
    cnorm[(size_t)bh * Cpad + m] = m < C ? (float)t : INFINITY;
    if (m == 0) amb_cnt[bh] = 0;
  }
}

// ---------------------------------------------------------------------------
// assign (tcgen05)
// ---------------------------------------------------------------------------
// One CTA per (head, run of pairs of token tiles), one CTA per SM:
//   warps 0-3 / 4-7  one thread per token of tile 0 / 1 of the current pair: scores of
//                    each centroid tile from TMEM, the two best scores and the best index;
//   warp 8           TMA: the pair's two token tiles, then its centroid tiles (hi and lo
//                    pieces) through a two-stage ring that both tiles read and that runs
//                    on across the pairs of the run;
//   warps 9 / 10     MMA issuer of tile 0 / 1: S = X C_hi^T + X C_lo^T into the tile's
//                    next logit buffer (two per tile, 128 columns each).
// The token tiles of the next pair load as soon as both issuers are done with the
// current ones and every row thread has read its token's norm.
template <int D>
struct AGeom {
  static constexpr int SUB = D / 64;
  static constexpr int XT = TT * D * 2;       // one token tile (bf16)
  static constexpr int CT = TCN * D * 2;      // one centroid piece tile (bf16)
  static constexpr int NCS = 2;               // centroid stages
  static constexpr int OFF_X = 0;             // [2 tiles][SUB][128 rows x 128 B]
  static constexpr int OFF_C = 2 * XT;        // [NCS][2 pieces][SUB][128 rows x 128 B]
  static constexpr int OFF_CTL = OFF_C + NCS * 2 * CT;
  static constexpr int OFF_CN = OFF_CTL + 256;  // [Cpad] ||c||^2, sized at launch
  static constexpr int TCOLS = 512;           // [2 tiles][2 buffers][128 columns]
  // one CTA per SM, so that its 512 TMEM columns are always free
  static constexpr int FLOOR = 232448 / 2 + 1024;
  static int smem(int Cpad) {
    const int need = OFF_CN + Cpad * 4 + 1024;  // + alignment slack
    return need > FLOOR ? need : FLOOR;
  }
};

struct ACtl {
  uint64_t x_full, x_empty, c_full[2], c_empty[2], s_full[2][2], s_free[2][2], done;
  uint32_t tmem_base;
  int abort;
};

struct AParams {
  CUtensorMap tmX, tmC;
  const float* cnorm;
  int32_t* labels;
  int32_t* amb_list;
  int32_t* amb_cnt;
  int32_t* err_flag;
  int N, Cpad, npair, run, nrun;
};

template <int D>
__global__ void __launch_bounds__(352, 1) assign_kernel(const __grid_constant__ AParams p) {
  using G = AGeom<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t base = smem_u32(smem);
  ACtl& c = *reinterpret_cast<ACtl*>(smem + G::OFF_CTL);
  auto bar = [&](uint64_t& b) { return smem_u32(&b); };
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int run = blockIdx.x % p.nrun, bh = blockIdx.x / p.nrun;
  const int pr0 = run * p.run;
  const int np = min(p.run, p.npair - pr0);  // pairs of this CTA
  const int ntc = p.Cpad / TCN;

  if (tid == 0) {
    tc::mbar_init(bar(c.x_full), 1);
    tc::mbar_init(bar(c.x_empty), 2 + 2 * TT);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(c.c_full[b]), 1);
      tc::mbar_init(bar(c.c_empty[b]), 2);
      for (int g = 0; g < 2; ++g) {
        tc::mbar_init(bar(c.s_full[g][b]), 1);
        tc::mbar_init(bar(c.s_free[g][b]), TT);
      }
    }
    tc::mbar_init(bar(c.done), 2);
    c.abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == 9) {
    tc::tmem_alloc(smem_u32(&c.tmem_base), G::TCOLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  tc::Waiter wt{&c.abort, p.err_flag, kWaitLimit};

  if (warp < 8) {
    // ============ rows: nearest centroids of one token of tile g ============
    const int g = warp / 4, row = tid & (TT - 1);
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    auto uni = [](bool x) { return __all_sync(0xffffffffu, x); };
    // the head's ||c||^2 into shared memory once (the eight row warps, then their barrier)
    float* cn = reinterpret_cast<float*>(smem + G::OFF_CN);
    float* red = reinterpret_cast<float*>(smem + G::OFF_CTL + 128);  // [8] warp maxima
    float cm = 0.f;  // largest ||c||^2 of the head (real centroids only)
    for (int m = tid; m < p.Cpad; m += 2 * TT) {
      const float v = __ldg(p.cnorm + (size_t)bh * p.Cpad + m);
      cn[m] = v;
      if (v < INFINITY) cm = fmaxf(cm, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    if (lane == 0) red[warp] = cm;
    asm volatile("bar.sync 1, %0;\n" ::"r"(2 * TT) : "memory");
    float cmax2 = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) cmax2 = fmaxf(cmax2, red[w]);
    bool ok = true;
    for (int i = 0; i < np && ok; ++i) {
      const int r = (pr0 + i) * 2 * TT + g * TT + row;  // the token
      ok = uni(wt.wait(bar(c.x_full), i & 1, 1));
      if (!ok) break;
      // ||x||^2 from the swizzled token tile (bf16 values, exact products in fp32)
      float xn = 0.f;
      const uint8_t* xt = smem + G::OFF_X + g * G::XT;
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint32_t off = (ch >> 3) * TT * 128 + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        const uint4 w = *reinterpret_cast<const uint4*>(xt + off);
        const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf16_lo(v[e]), b = bf16_hi(v[e]);
          xn = fmaf(a, a, fmaf(b, b, xn));
        }
      }
      tc::mbar_arrive(bar(c.x_empty));  // this thread is done with the token tiles
      float best = INFINITY, second = INFINITY;
      int bi = 0;
      for (int t = 0; t < ntc && ok; ++t) {
        const int T = i * ntc + t, b = T & 1;
        ok = uni(wt.wait(bar(c.s_full[g][b]), (T >> 1) & 1, 2));
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t scol = tmem + lane_off + 256 * g + TCN * b;
#pragma unroll 1
        for (int h = 0; h < TCN / 64; ++h) {
          uint32_t sr[64];
          tc::tmem_ld32(scol + 64 * h, sr);
          tc::tmem_ld32(scol + 64 * h + 32, sr + 32);
          tc::tmem_wait_ld();
          if (h == TCN / 64 - 1) {
            tc::fence_before_sync();
            tc::mbar_arrive(bar(c.s_free[g][b]));
          }
          const int m0 = t * TCN + 64 * h;
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            const float4 n4 = *reinterpret_cast<const float4*>(cn + m0 + e);
            const float nv[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const float s = fmaf(-2.f, __uint_as_float(sr[e + f]), nv[f]);
              // the two best scores and the best index (the first on ties)
              bi = s < best ? m0 + e + f : bi;
              second = fminf(second, fmaxf(best, s));
              best = fminf(best, s);
            }
          }
        }
      }
      if (ok && r < p.N) {
        // Error bound of one fp32 score here: the pieces hold c to 2^-17 relative, the
        // products accumulate in fp32 over 2d terms, ||c||^2 and the final fma round
        // once: |err| <= 5e-5 |x| |c| + 1.2e-7 |c|^2. A token whose two best scores are
        // closer than twice that (with 20% to spare) is decided in fp64 instead.
        const float xa = sqrtf(xn), ca = sqrtf(cmax2);
        const float thr = 1.2e-4f * xa * ca + 3e-7f * cmax2;
        p.labels[(size_t)bh * p.N + r] = bi;
        if (!(second - best > thr)) {
          const int k = atomicAdd(p.amb_cnt + bh, 1);  // undecided: recheck in fp64
          p.amb_list[(size_t)bh * p.N + k] = r;
        }
      }
    }
  } else if (warp == 8) {
    // ======================== TMA producer ========================
    if (lane == 0) {
      bool ok = true;
      uint32_t used = 0, par = 0;  // per centroid stage: loaded, parity of the last load
      int xloads = 0;
      for (int i = 0; i < np && ok; ++i) {
        if (i >= 1) ok = wt.wait(bar(c.x_empty), (i - 1) & 1, 7);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar(c.x_full), 2 * G::XT);
        for (int g = 0; g < 2; ++g)
          for (int x = 0; x < G::SUB; ++x)
            tc::tma_load_3d(base + G::OFF_X + g * G::XT + x * TT * 128, &p.tmX, bar(c.x_full),
                            64 * x, (pr0 + i) * 2 * TT + g * TT, bh);
        ++xloads;
        for (int t = 0; t < ntc && ok; ++t) {
          const int T = i * ntc + t, st = T & 1, ph = (T >> 1) & 1;
          if (T >= 2) ok = wt.wait(bar(c.c_empty[st]), ph ^ 1, 3);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(bar(c.c_full[st]), 2 * G::CT);
          for (int pc = 0; pc < 2; ++pc)
            for (int x = 0; x < G::SUB; ++x)
              tc::tma_load_3d(base + G::OFF_C + (st * 2 + pc) * G::CT + x * TCN * 128, &p.tmC,
                              bar(c.c_full[st]), 64 * x, t * TCN, 2 * bh + pc);
          used |= 1u << st;
          par = (par & ~(1u << st)) | ((uint32_t)ph << st);
        }
      }
      // every load issued lands before the CTA exits
      if (xloads > 0) tc::wait_drain(bar(c.x_full), (xloads - 1) & 1, kWaitLimit);
      for (int st = 0; st < 2; ++st)
        if ((used >> st) & 1) tc::wait_drain(bar(c.c_full[st]), (par >> st) & 1, kWaitLimit);
    }
  } else if (warp == 9 || warp == 10) {
    // ================ MMA issuers: warp 9 + g for token tile g ================
    if (lane == 0) {
      constexpr uint32_t I_S = tc::idesc_f16(1, 1, 0, TCN);
      const int g = warp - 9;
      const uint64_t dx = tc::sdesc(base + G::OFF_X + g * G::XT, 16, 1024);
      bool ok = true;
      for (int i = 0; i < np && ok; ++i) {
        ok = wt.wait(bar(c.x_full), i & 1, 4);
        for (int t = 0; t < ntc && ok; ++t) {
          const int T = i * ntc + t, b = T & 1, st = T & 1;
          ok = wt.wait(bar(c.c_full[st]), (T >> 1) & 1, 5) &&
               (T < 2 || wt.wait(bar(c.s_free[g][b]), ((T >> 1) - 1) & 1, 6));
          if (!ok) break;
          tc::fence_after_sync();
          const uint64_t dc = tc::sdesc(base + G::OFF_C + st * 2 * G::CT, 16, 1024);
          for (int pc = 0; pc < 2; ++pc) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t aoff = ((kk / 4) * TT * 128 + (kk % 4) * 32) >> 4;
              const uint32_t boff = (pc * G::CT + (kk / 4) * TCN * 128 + (kk % 4) * 32) >> 4;
              tc::mma_ss(tmem + 256 * g + TCN * b, dx + aoff, dc + boff, I_S, (pc | kk) > 0);
            }
          }
          tc::mma_commit(bar(c.s_full[g][b]));
          tc::mma_commit(bar(c.c_empty[st]));
        }
        if (ok) tc::mma_commit(bar(c.x_empty));  // the token tiles are read
      }
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

// ---------------------------------------------------------------------------
// recheck: the undecided tokens in fp64, one CTA per token
// ---------------------------------------------------------------------------
// dist_m = sum_i (x_i - c_mi)^2, lane l summing dimensions l, l+32, ... in order and the
// lanes combined by a fixed butterfly. Warp w takes the centroids m = w, w + 8, ...; the
// smallest distance wins, ties to the lowest index.
constexpr int kRecheckWarps = 8;

__device__ __forceinline__ double dist64(const double* xv, const double* cm, int d, int lane) {
  double s = 0.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (lane + 32 * k < d) {
      const double t = xv[k] - cm[lane + 32 * k];
      s = fma(t, t, s);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

__global__ void __launch_bounds__(32 * kRecheckWarps)
recheck_kernel(const uint16_t* __restrict__ x, const double* __restrict__ cent, int N, int d,
               int C, const int32_t* __restrict__ amb_list, const int32_t* __restrict__ amb_cnt,
               int32_t* __restrict__ labels) {
  __shared__ double wbest[kRecheckWarps];
  __shared__ int wbi[kRecheckWarps];
  const int bh = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int cnt = amb_cnt[bh];
  const double* cb = cent + (size_t)bh * C * d;
  for (int e = blockIdx.x; e < cnt; e += gridDim.x) {
    const int r = amb_list[(size_t)bh * N + e];
    const uint16_t* xr = x + ((size_t)bh * N + r) * d;
    double xv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      xv[k] = lane + 32 * k < d ? (double)__uint_as_float((uint32_t)xr[lane + 32 * k] << 16) : 0.0;
    double best = INFINITY;
    int bi = 0;
    int m = warp;
    for (; m + kRecheckWarps < C; m += 2 * kRecheckWarps) {  // two centroids in flight
      const double s0 = dist64(xv, cb + (size_t)m * d, d, lane);
      const double s1 = dist64(xv, cb + (size_t)(m + kRecheckWarps) * d, d, lane);
      if (s0 < best) { best = s0; bi = m; }
      if (s1 < best) { best = s1; bi = m + kRecheckWarps; }
    }
    if (m < C) {
      const double s0 = dist64(xv, cb + (size_t)m * d, d, lane);
      if (s0 < best) { best = s0; bi = m; }
    }
    if (lane == 0) {
      wbest[warp] = best;
      wbi[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double b = wbest[0];
      int ib = wbi[0];
      for (int w = 1; w < kRecheckWarps; ++w)
        if (wbest[w] < b || (wbest[w] == b && wbi[w] < ib)) {
          b = wbest[w];
          ib = wbi[w];
        }
      labels[(size_t)bh * N + r] = ib;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// stable counting sort of the labels
// ---------------------------------------------------------------------------
// counts[bh][chunk][m]: members of cluster m among the chunk's tokens.
__global__ void hist_kernel(const int32_t* __restrict__ labels, int N, int C, int nchunk,
                            int32_t* __restrict__ counts) {
  extern __shared__ int32_t hsm[];  // [kSortWarps][C]
  const int bh = blockIdx.y, w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kSortWarps + w;
  int32_t* h = hsm + w * C;
  for (int m = lane; m < C; m += 32) h[m] = 0;
  __syncwarp();
  if (chunk < nchunk) {
    const int s = chunk * kChunk, e = min(N, s + kChunk);
    for (int r = s + lane; r < e; r += 32) atomicAdd(h + labels[(size_t)bh * N + r], 1);
  }
  __syncwarp();
  if (chunk < nchunk)
    for (int m = lane; m < C; m += 32) counts[((size_t)bh * nchunk + chunk) * C + m] = h[m];
}

// offsets[m] = members of clusters < m; counts becomes the first position of each
// (chunk, cluster) pair: offsets[m] + members of m in earlier chunks.
__global__ void scan_kernel(int32_t* __restrict__ counts, int C, int nchunk,
                            int32_t* __restrict__ offsets, int32_t* __restrict__ seg_off) {
  extern __shared__ int32_t ssm[];  // [C] totals
  const int bh = blockIdx.x;
  int32_t* cnt = counts + (size_t)bh * nchunk * C;
  for (int m = threadIdx.x; m < C; m += blockDim.x) {
    int run = 0;
    for (int k = 0; k < nchunk; ++k) {
      const int v = cnt[(size_t)k * C + m];
      cnt[(size_t)k * C + m] = run;
      run += v;
    }
    ssm[m] = run;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, sacc = 0;  // members, and segments of kSeg members, of clusters < m
    for (int m = 0; m < C; ++m) {
      const int v = ssm[m];
      ssm[m] = acc;
      seg_off[(size_t)bh * (C + 1) + m] = sacc;
      acc += v;
      sacc += (v + kSeg - 1) / kSeg;
    }
    offsets[(size_t)bh * (C + 1) + C] = acc;
    seg_off[(size_t)bh * (C + 1) + C] = sacc;
  }
  __syncthreads();
  for (int m = threadIdx.x; m < C; m += blockDim.x) {
    const int o = ssm[m];
    offsets[(size_t)bh * (C + 1) + m] = o;
    for (int k = 0; k < nchunk; ++k) cnt[(size_t)k * C + m] += o;
  }
}

// Each warp walks its chunk 32 tokens at a time, in token order: lanes holding the same
// label take consecutive positions in lane order after that label's cursor.
__global__ void scatter_kernel(const int32_t* __restrict__ labels, int N, int C, int nchunk,
                               const int32_t* __restrict__ starts, int32_t* __restrict__ perm) {
  extern __shared__ int32_t csm[];  // [kSortWarps][C] cursors
  const int bh = blockIdx.y, w = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x * kSortWarps + w;
  if (chunk >= nchunk) return;
  int32_t* cur = csm + w * C;
  for (int m = lane; m < C; m += 32) cur[m] = starts[((size_t)bh * nchunk + chunk) * C + m];
  __syncwarp();
  const int s = chunk * kChunk, e = min(N, s + kChunk);
  const unsigned lt = (1u << lane) - 1u;
  for (int r0 = s; r0 < e; r0 += 32) {
    const int r = r0 + lane;
    const bool valid = r < e;
    const unsigned act = __ballot_sync(0xffffffffu, valid);
    const int lab = valid ? labels[(size_t)bh * N + r] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, lab) & act;
    int base = 0;
    if (valid) base = cur[lab];  // every peer reads the cursor before the leader moves it
    __syncwarp();
    if (valid) {
      perm[(size_t)bh * N + base + __popc(peers & lt)] = r;
      if ((peers & lt) == 0) cur[lab] = base + __popc(peers);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// update: each centroid to the fp64 mean of its members; one without members stays
// ---------------------------------------------------------------------------
// The sorted members are cut into segments of at most kSeg per cluster (the scan gives
// each cluster's first segment), so that a very large cluster does not run on one CTA:
// one CTA sums each segment, then one CTA per cluster adds its segments in order. Every
// sum of bf16 values here is exact in fp64, so the split changes no bit of the means.
// Segment CTA: 512 threads, d / 8 per member row (eight dimensions each, one 16-byte
// load), 512 / (d / 8) member rows side by side, combined in a fixed order.
constexpr int kUpdThreads = 512;

__global__ void __launch_bounds__(kUpdThreads)
segment_sum_kernel(const uint16_t* __restrict__ x, int N, int d, int C, int maxseg,
                   const int32_t* __restrict__ perm, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ seg_off, double* __restrict__ part) {
  __shared__ double lanes_sum[kUpdThreads * 8];  // [row lane][d]
  const int sg = blockIdx.x, bh = blockIdx.y;
  const int32_t* so = seg_off + (size_t)bh * (C + 1);
  if (sg >= so[C]) return;
  // the segment's cluster: the last m with so[m] <= sg
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (so[mid] <= sg) lo = mid; else hi = mid - 1;
  }
  const int m = lo;
  const int32_t* of = offsets + (size_t)bh * (C + 1);
  const int s = of[m] + (sg - so[m]) * kSeg, e = min(s + kSeg, of[m + 1]);
  const int cpr = d / 8, lanes = kUpdThreads / cpr;
  const int rl = threadIdx.x / cpr, ch = threadIdx.x % cpr;
  const int32_t* pr = perm + (size_t)bh * N;
  const uint16_t* xb = x + (size_t)bh * N * d + ch * 8;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int k = s + rl; k < e; k += lanes) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(xb + (size_t)__ldg(pr + k) * d));
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc[2 * q] += (double)bf16_lo(v[q]);
      acc[2 * q + 1] += (double)bf16_hi(v[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) lanes_sum[rl * d + ch * 8 + q] = acc[q];
  __syncthreads();
  if (threadIdx.x < d) {
    double sum = 0.0;
    for (int l = 0; l < lanes; ++l) sum += lanes_sum[l * d + threadIdx.x];
    part[((size_t)bh * maxseg + sg) * d + threadIdx.x] = sum;
  }
}

__global__ void combine_kernel(int d, int C, int maxseg, const int32_t* __restrict__ offsets,
                               const int32_t* __restrict__ seg_off,
                               const double* __restrict__ part, double* __restrict__ cent) {
  const int m = blockIdx.x, bh = blockIdx.y, i = threadIdx.x;
  const int32_t* of = offsets + (size_t)bh * (C + 1);
  const int32_t* so = seg_off + (size_t)bh * (C + 1);
  const int cnt = of[m + 1] - of[m];
  if (cnt == 0 || i >= d) return;  // no members: the centroid stays
  double sum = 0.0;
  for (int sg = so[m]; sg < so[m + 1]; ++sg) sum += part[((size_t)bh * maxseg + sg) * d + i];
  cent[((size_t)bh * C + m) * d + i] = sum / (double)cnt;
}

// ---------------------------------------------------------------------------
// row permutations
// ---------------------------------------------------------------------------
// dst[p] = src[perm[p]] (gather) or dst[perm[p]] = src[p] (scatter), rows of row_bytes
// (a multiple of 16), 16 bytes per thread step.
template <bool GATHER>
__global__ void permute_kernel(const uint8_t* __restrict__ src, const int32_t* __restrict__ perm,
                               int N, int row_bytes, long long total_vec, uint8_t* __restrict__ dst) {
  const int vpr = row_bytes / 16;
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < total_vec;
       v += (long long)gridDim.x * blockDim.x) {
    const long long row = v / vpr;
    const int col = (int)(v % vpr);
    const long long other = (row / N) * N + perm[row];
    const long long from = GATHER ? other : row, to = GATHER ? row : other;
    reinterpret_cast<uint4*>(dst + to * row_bytes)[col] =
        reinterpret_cast<const uint4*>(src + from * row_bytes)[col];
  }
}

}  // namespace km

namespace {

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

template <int D>
cudaError_t assign_t(const KmeansArgs& a, int Cpad, cudaStream_t st) {
  using G = km::AGeom<D>;
  km::AParams p;
  const uint64_t bh = (uint64_t)a.B * a.H;
  if (!map3d(&p.tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x, D, a.N, bh, km::TT) ||
      !map3d(&p.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.pieces, D, Cpad, 2 * bh, km::TCN))
    return cudaErrorInvalidValue;
  p.cnorm = a.cnorm;
  p.labels = a.labels;
  p.amb_list = a.amb_list;
  p.amb_cnt = a.amb_cnt;
  p.err_flag = a.err_flag;
  p.N = a.N;
  p.Cpad = Cpad;
  p.npair = km::cdiv(a.N, 2 * km::TT);
  // pairs per CTA: the run length that minimises waves x (run + 1/2), one CTA per SM and
  // the CTA's setup costed as half a pair
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 1;
  double best_cost = 1e300;
  p.run = 1;
  for (int run = 1; run <= 32; ++run) {
    const double ctas = (double)bh * km::cdiv(p.npair, run);
    const double cost = std::ceil(ctas / sms) * (run + 0.5);
    if (cost < best_cost) {
      best_cost = cost;
      p.run = run;
    }
    if (run >= p.npair) break;
  }
  p.nrun = km::cdiv(p.npair, p.run);
  auto kern = km::assign_kernel<D>;
  const int smem = G::smem(Cpad);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(p.nrun * bh), 352, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Scratch for sparse_attn_kmeans_noalloc: one fixed buffer per device, part of the
// module's global memory (no allocation at call time).
static __device__ __align__(256) uint8_t g_kmeans_scratch[kKmeansScratchBytes];

// The buffer's device address on the current device. Looked up on every call: the
// lookup costs microseconds, and an address kept across calls would go stale if the
// device's context were reset (the module, and with it the buffer, is then loaded
// again). On failure the runtime's error state is cleared, so that it does not
// surface in a later launch check, and the error is returned.
cudaError_t kmeans_scratch(void** addr) {
  *addr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(addr, g_kmeans_scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *addr = nullptr;
  }
  return e;
}

// Where each work buffer of launch_kmeans sits in cwork and iwork (byte offsets);
// the sizes the caller allocates are the two ends, so the carving and the sizes
// cannot disagree.
KmeansLayout kmeans_layout(int B, int H, int N, int d, int C) {
  const size_t bh = (size_t)B * H;
  const size_t Cpad = (size_t)km::cdiv(C, km::TCN) * km::TCN, nchunk = km::cdiv(N, km::kChunk);
  const size_t maxseg = (size_t)km::cdiv(N, km::kSeg) + C;
  KmeansLayout L;
  L.pieces = 0;                                                // [bh][2][Cpad][d] bf16
  L.cnorm = L.pieces + align256(bh * 2 * Cpad * d * 2);        // [bh][Cpad] fp32
  L.part = L.cnorm + align256(bh * Cpad * 4);                  // [bh][maxseg][d] fp64
  L.cwork_end = L.part + bh * maxseg * d * 8;
  L.counts = 0;                                                // [bh][nchunk][C] int32
  L.amb_list = L.counts + align256(bh * nchunk * C * 4);       // [bh][N] int32
  L.amb_cnt = L.amb_list + align256(bh * N * 4);               // [bh] int32
  L.seg_off = L.amb_cnt + align256(bh * 4);                    // [bh][C + 1] int32
  L.iwork_end = L.seg_off + bh * (C + 1) * 4;
  return L;
}

void kmeans_sizes(int B, int H, int N, int d, int C, size_t sizes[3]) {
  const KmeansLayout L = kmeans_layout(B, H, N, d, C);
  sizes[0] = (size_t)B * H * C * d * sizeof(double);
  sizes[1] = L.cwork_end;
  sizes[2] = L.iwork_end;
}

cudaError_t launch_kmeans(const KmeansArgs& in, cudaStream_t st) {
  KmeansArgs a = in;
  const int bh = a.B * a.H, C = a.C, d = a.d, N = a.N;
  const int Cpad = km::cdiv(C, km::TCN) * km::TCN, nchunk = km::cdiv(N, km::kChunk);
  // carve the work buffers
  const int maxseg = km::cdiv(N, km::kSeg) + C;
  const KmeansLayout L = kmeans_layout(a.B, a.H, N, d, C);
  uint8_t* cw = reinterpret_cast<uint8_t*>(a.cwork);
  uint8_t* iw = reinterpret_cast<uint8_t*>(a.iwork);
  a.pieces = reinterpret_cast<uint16_t*>(cw + L.pieces);
  a.cnorm = reinterpret_cast<float*>(cw + L.cnorm);
  double* part = reinterpret_cast<double*>(cw + L.part);
  a.counts = reinterpret_cast<int32_t*>(iw + L.counts);
  a.amb_list = reinterpret_cast<int32_t*>(iw + L.amb_list);
  a.amb_cnt = reinterpret_cast<int32_t*>(iw + L.amb_cnt);
  int32_t* seg_off = reinterpret_cast<int32_t*>(iw + L.seg_off);

  const int sort_smem = km::kSortWarps * C * 4;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(km::hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                sort_smem)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(km::scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                sort_smem)) != cudaSuccess)
    return e;
  const dim3 gsort(km::cdiv(nchunk, km::kSortWarps), bh);
  auto assign = [&]() -> cudaError_t {
    cudaError_t r = d == 64 ? assign_t<64>(a, Cpad, st) : assign_t<128>(a, Cpad, st);
    if (r != cudaSuccess) return r;
    km::recheck_kernel<<<dim3(256, bh), 32 * km::kRecheckWarps, 0, st>>>(
        a.x, a.cent, N, d, C, a.amb_list, a.amb_cnt, a.labels);
    return cudaGetLastError();
  };
  auto sort = [&]() -> cudaError_t {
    km::hist_kernel<<<gsort, 32 * km::kSortWarps, sort_smem, st>>>(a.labels, N, C, nchunk,
                                                                   a.counts);
    km::scan_kernel<<<bh, 256, C * 4, st>>>(a.counts, C, nchunk, a.offsets, seg_off);
    km::scatter_kernel<<<gsort, 32 * km::kSortWarps, sort_smem, st>>>(a.labels, N, C, nchunk,
                                                                      a.counts, a.perm);
    return cudaGetLastError();
  };
  auto prep = [&]() -> cudaError_t {
    km::prep_kernel<<<dim3(Cpad, bh), 64, 0, st>>>(a.cent, C, Cpad, d, a.pieces, a.cnorm,
                                                  a.amb_cnt);
    return cudaGetLastError();
  };
  km::init_kernel<<<dim3(C, bh), 64, 0, st>>>(a.x, N, d, C, a.cent);
  if ((e = prep()) != cudaSuccess) return e;
  for (int t = 0; t < a.iters; ++t) {
    if ((e = assign()) != cudaSuccess) return e;
    if ((e = sort()) != cudaSuccess) return e;
    km::segment_sum_kernel<<<dim3(maxseg, bh), km::kUpdThreads, 0, st>>>(
        a.x, N, d, C, maxseg, a.perm, a.offsets, seg_off, part);
    km::combine_kernel<<<dim3(C, bh), d, 0, st>>>(d, C, maxseg, a.offsets, seg_off, part, a.cent);
    if ((e = prep()) != cudaSuccess) return e;
  }
  if ((e = assign()) != cudaSuccess) return e;
  return sort();
}

cudaError_t launch_permute_rows(const PermuteArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.B * a.H * a.N;
  const long long total = rows * (a.row_bytes / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long want = (total + threads - 1) / threads;
  const unsigned blocks = (unsigned)(want < 148LL * 64 ? want : 148LL * 64);
  if (a.gather)
    km::permute_kernel<true><<<blocks, threads, 0, st>>>(
        reinterpret_cast<const uint8_t*>(a.src), a.perm, a.N, a.row_bytes, total,
        reinterpret_cast<uint8_t*>(a.dst));
  else
    km::permute_kernel<false><<<blocks, threads, 0, st>>>(
        reinterpret_cast<const uint8_t*>(a.src), a.perm, a.N, a.row_bytes, total,
        reinterpret_cast<uint8_t*>(a.dst));
  return cudaGetLastError();
}

}  // namespace sa
