// Routing from pooled scores, and the structured (window + rotating anchor) mask.
//
// Routing follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient
// Diffusion Transformers" §2 (top-k choice of the critical blocks S_i) with the
// pooled proxies of "SVG-EAR" §2 B (query-block centroids stand in for the
// block's queries). The structured mask follows "LVSA: Training-Free Sparse
// Attention for Long Video Diffusion" §2 (A(t) = G u W(t), anchors shifted by
// s mod T_per).
//
// Route kernel: one CTA of 8 warps per (batch*head, R query blocks), R = 16 (8 when a
// row holds more than 1024 key blocks).
//   1. Scores s_ij = scale * qbar_i . kbar_j in fp32 for the CTA's R rows. The head's
//      dim-major centroid table streams through shared memory in chunks of KD rows (KD
//      dimensions, all key blocks of each): KD consecutive rows are one contiguous range
//      that starts on a 16-byte boundary, copied with 16-byte cp.async into a double
//      buffer; each thread accumulates an 8-row x MC-column tile with fp32 FMAs, the 8
//      rows' qbar values broadcast from shared memory. Every score is one fma chain over
//      d = 0 .. D-1 in order.
//   2. One warp per query block selects (select_row) over order-preserving score keys
//      held in registers: the threshold is found a byte at a time from warp histograms
//      (top-k) or by a 32-step bit search on the covered mass (mass rule), ties at the
//      threshold are taken in ascending block index, and the kept indices are written in
//      ascending order with ballots.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace sa {

constexpr int kRouteThreads = 256;


// One warp selects the kept blocks of one query block from its scores s[0..nkb).
// Lane l holds blocks j = l + 32 i (i < SLOTS) as order-preserving 32-bit keys.
//   1. The threshold key T:
//        top-k: the largest T with #{key >= T} >= k, found one byte at a time (most
//               significant first) from a 256-bin histogram of the keys that match the
//               bytes found so far (warp-private bins in shared memory, integer counts);
//        mass:  the largest T with sum_{key >= T} e^(s - max) >= tau * Z, by an MSB-first
//               search over the 32 key bits (masses summed in one fixed order).
//   2. Every block with key > T is kept; blocks with key == T (ties) are taken in
//      ascending j until the count (top-k) or the mass (mass rule) is reached, so the
//      order is (score descending, index ascending).
//   3. Kept indices are written in ascending j with ballots.
template <int SLOTS, int MODE>
SA_DEVI void select_row(const float* s, int nkb, int keep, float tau, int32_t* out,
                        int32_t* cnt_out, int cap, int lane, int* hist) {
  uint32_t key[SLOTS];
  float e[MODE == 1 ? SLOTS : 1];
#pragma unroll
  for (int i = 0; i < SLOTS; ++i) {
    const int j = lane + 32 * i;
    key[i] = j < nkb ? float_key(s[j]) : 0u;  // 0 sorts below every real score
  }
  float goal = 0.f;
  uint32_t T = 0;
  int above = 0;        // top-k: keys strictly above T
  float mabove = 0.f;   // mass: their mass
  if constexpr (MODE == 0) {
    uint32_t pmask = 0;
    int need = keep;  // keys >= T still to be found among those matching the prefix
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int t = 0; t < 8; ++t) hist[lane * 8 + t] = 0;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < SLOTS; ++i)
        if (lane + 32 * i < nkb && (key[i] & pmask) == T) atomicAdd(&hist[(key[i] >> shift) & 255], 1);
      __syncwarp();
      // lane l holds bins 255 - 8 l - t (t = 0..7), i.e. digits in descending order
      int cnt[8], tot = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        cnt[t] = hist[255 - 8 * lane - t];
        tot += cnt[t];
      }
      int incl = tot;  // inclusive scan over lanes (higher digits first)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int before = incl - tot;  // keys with a higher digit than this lane's bins
      // the digit where the count from the top first reaches `need`
      int found = -1, above_d = 0, bucket = 0;
      if (before < need && incl >= need) {
        int acc = before;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (found < 0 && acc + cnt[t] >= need) {
            found = 255 - 8 * lane - t;
            above_d = acc;
            bucket = cnt[t];
          }
          acc += cnt[t];
        }
      }
      const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
      const int src = __ffs(who) - 1;
      found = __shfl_sync(0xffffffffu, found, src);
      above_d = __shfl_sync(0xffffffffu, above_d, src);
      bucket = __shfl_sync(0xffffffffu, bucket, src);
      T |= (uint32_t)found << shift;
      pmask |= 255u << shift;
      need -= above_d;
      above += above_d;
      __syncwarp();  // the bins are read before the next pass clears them
      if (shift > 0 && (need == 1 || need == bucket)) {
        // The rest follows without more passes: the `bucket` keys that match the prefix
        // found so far hold the threshold. One still to find: it is their largest; all
        // of them needed: it is their smallest, and those above it count as above T.
        const bool top = need == 1;
        uint32_t ext = top ? 0u : 0xffffffffu;
#pragma unroll
        for (int i = 0; i < SLOTS; ++i)
          if (lane + 32 * i < nkb && (key[i] & pmask) == T) ext = top ? max(ext, key[i]) : min(ext, key[i]);
        T = top ? __reduce_max_sync(0xffffffffu, ext) : __reduce_min_sync(0xffffffffu, ext);
        if (!top) {
          int eq = 0;
#pragma unroll
          for (int i = 0; i < SLOTS; ++i) eq += (lane + 32 * i < nkb && key[i] == T) ? 1 : 0;
          above += bucket - (int)__reduce_add_sync(0xffffffffu, (unsigned)eq);
        }
        break;
      }
    }
  } else {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < SLOTS; ++i)
      if (lane + 32 * i < nkb) mx = fmaxf(mx, s[lane + 32 * i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) {
      e[i] = lane + 32 * i < nkb ? expf(s[lane + 32 * i] - mx) : 0.f;
      z += e[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    goal = tau * z;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = T | (1u << bit);
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < SLOTS; ++i) m += key[i] >= cand ? e[i] : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
      if (m >= goal) T = cand;
    }
    // what the strictly larger keys already give
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) mabove += key[i] > T ? e[i] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mabove += __shfl_xor_sync(0xffffffffu, mabove, o);
  }
  // walk the ties in ascending j; write every kept index in ascending j
  const unsigned lt = (1u << lane) - 1u;
  int off = 0, ties = 0;
  float tmass = 0.f;
  bool done = false;  // the tie quota is filled
#pragma unroll
  for (int i = 0; i < SLOTS; ++i) {
    const bool tie = key[i] == T && lane + 32 * i < nkb;
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    bool take_tie = false;
    if constexpr (MODE == 0) {
      take_tie = tie && (ties + __popc(tb & lt)) < keep - above;
      ties += __popc(tb);
    } else {
      // inclusive prefix of tie masses in j order
      float x = tie ? e[i] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const float before = tmass + x - (tie ? e[i] : 0.f);
      take_tie = tie && !done && (mabove + before < goal);
      tmass += __shfl_sync(0xffffffffu, x, 31);
      done = done || (mabove + tmass >= goal);
    }
    const bool in = key[i] > T || take_tie;
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (in) {
      const int pos = off + __popc(bal & lt);
      if (pos < cap) out[pos] = lane + 32 * i;
    }
    off += __popc(bal);
  }
  if (lane == 0) *cnt_out = min(off, cap);
}

// Shared-memory layout of one route CTA, in floats: the qbar block [D][R]; two chunk
// buffers, each KD rows of the centroid table (KD * nkb floats, contiguous as in global
// memory) and NKP - nkb spare floats that the column threads past nkb read (their
// columns are never stored); the score rows [R][nkb], over the chunk buffers once the
// scoring is done; a 256-bin histogram per warp for the top-k selection.
template <int D, int RG, int MC, int KD>
struct RouteSmem {
  static constexpr int R = 8 * RG, CT = kRouteThreads / RG, NKP = CT * MC;
  static size_t __host__ __device__ buf(int nkb) { return ((size_t)KD * nkb + (NKP - nkb) + 3) & ~(size_t)3; }
  static size_t __host__ __device__ chunks(int nkb) {
    const size_t a = 2 * buf(nkb), b = (size_t)R * nkb;
    return a > b ? a : b;
  }
  static size_t __host__ __device__ bytes(int nkb) {
    return ((size_t)D * R + chunks(nkb) + (kRouteThreads / 32) * 256) * 4;
  }
};

template <int D, int SLOTS, int RG, int MC, int KD, int MODE>
__global__ void __launch_bounds__(kRouteThreads, SLOTS <= 32 ? 2 : 1)
route_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar_t, int nqb, int nkb,
             int keep, float tau, float scale, int32_t* __restrict__ kv_idx,
             int32_t* __restrict__ kv_cnt, int cap, const float* __restrict__ cov,
             const float* __restrict__ pre) {
  using L = RouteSmem<D, RG, MC, KD>;
  constexpr int R = L::R, CT = L::CT;
  constexpr int NCH = D / KD;                // chunks of KD dimensions
  static_assert(D % KD == 0 && KD % 4 == 0, "a chunk is whole 16-byte pieces");
  extern __shared__ __align__(16) float rsm[];
  float* qs = rsm;                           // [D][R]: qs[c * R + r] = qbar of row r, dim c
  float* kc = qs + D * R;                    // [2] chunk buffers
  float* sc = kc;                            // [R][nkb] scores, once the chunks are done
  int* hist = reinterpret_cast<int*>(kc + L::chunks(nkb));  // [warps][256]
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int rows = min(R, nqb - i0);

  if (pre) {
    // precomputed scores (error-aware routing): the CTA's rows are one contiguous range,
    // copied with 4-byte cp.async (its start has no 16-byte alignment) so that every
    // thread's loads are in flight at once
    const float* src = pre + ((size_t)bh * nqb + i0) * nkb;
    const int n = rows * nkb;
    for (int x = tid; x < n; x += kRouteThreads) cp_async4(smem_u32(sc + x), src + x, 4);
    cp_async_commit();
    cp_async_wait<0>();
  } else {
    // Chunk ch: rows ch*KD .. ch*KD+KD-1 of the head's table, KD*nkb floats from element
    // (bh*D + ch*KD)*nkb, a multiple of 4 (D and KD are), so a 16-byte aligned range.
    const float* kt = kbar_t + (size_t)bh * D * nkb;
    const size_t bs = L::buf(nkb);
    const int pieces = KD * nkb / 4;
    auto load_chunk = [&](int ch, int b) {
      const float* src = kt + (size_t)ch * KD * nkb;
      float* dst = kc + b * bs;
      for (int x = tid; x < pieces; x += kRouteThreads) cp_async16(smem_u32(dst + 4 * x), src + 4 * x, 16);
      cp_async_commit();
    };
    load_chunk(0, 0);
    for (int x = tid; x < D * R; x += kRouteThreads) {
      const int r = x / D, c = x % D;   // coalesced along c
      qs[c * R + r] = r < rows ? qbar[((size_t)bh * nqb + i0 + r) * D + c] : 0.f;
    }
    const int rg = tid / CT, ct = tid % CT;   // a warp shares its group of 8 rows
    // acc[r][m]: row r of the group, column ct + CT m
    float acc[8][MC];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int m = 0; m < MC; ++m) acc[r][m] = 0.f;
    for (int ch = 0; ch < NCH; ++ch) {
      cp_async_wait<0>();
      __syncthreads();  // chunk ch (and the qbar block) visible; chunk ch-1 read by every thread
      if (ch + 1 < NCH) load_chunk(ch + 1, (ch + 1) & 1);  // into the buffer of chunk ch-1
      const float* kb = kc + (ch & 1) * bs + ct;
#pragma unroll
      for (int k = 0; k < KD; ++k) {
        const int c = ch * KD + k;
        const float4 q0 = *reinterpret_cast<const float4*>(qs + c * R + rg * 8);
        const float4 q1 = *reinterpret_cast<const float4*>(qs + c * R + rg * 8 + 4);
        const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int m = 0; m < MC; ++m) {
          const float kv = kb[k * nkb + CT * m];
#pragma unroll
          for (int r = 0; r < 8; ++r) acc[r][m] = fmaf(qv[r], kv, acc[r][m]);
        }
      }
    }
    __syncthreads();  // every chunk read before the scores overwrite the buffers
#pragma unroll
    for (int m = 0; m < MC; ++m) {
      const int j = ct + CT * m;
      if (j >= nkb) continue;
      // covariance-aware top-k: the log of block j's covariance norm joins every row's score
      const float bias = cov ? logf(cov[(size_t)bh * nkb + j]) : 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) sc[(rg * 8 + r) * nkb + j] = scale * acc[r][m] + bias;
    }
  }
  __syncthreads();

  const int warp = tid / 32, lane = tid % 32;
  for (int r = warp; r < rows; r += kRouteThreads / 32)
    select_row<SLOTS, MODE>(sc + r * nkb, nkb, keep, tau,
                            kv_idx + ((size_t)bh * nqb + i0 + r) * cap,
                            kv_cnt + (size_t)bh * nqb + i0 + r, cap, lane, hist + warp * 256);
}

template <int D, int SLOTS, int RG, int MC, int KD>
static cudaError_t launch_route_t(const RouteArgs& p, cudaStream_t st) {
  const size_t smem = RouteSmem<D, RG, MC, KD>::bytes(p.nkb);
  auto kern = p.mode == 0 ? route_kernel<D, SLOTS, RG, MC, KD, 0> : route_kernel<D, SLOTS, RG, MC, KD, 1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.nqb + 8 * RG - 1) / (8 * RG), p.B * p.H);
  kern<<<grid, kRouteThreads, smem, st>>>(p.qbar, p.kbar_t, p.nqb, p.nkb, p.keep, p.tau, p.scale,
                                          p.kv_idx, p.kv_cnt, p.cap, p.cov, p.scores);
  return cudaGetLastError();
}

// Key slots per lane (select_row) and columns per thread (scoring) from nkb: up to 1024
// key blocks, two groups of 8 rows share the columns (MC = ceil(nkb / 128)); beyond,
// one group of 8 rows (MC = ceil(nkb / 256)). Chunks of 8 dimensions while the chunk
// stays small, else 4.
template <int D>
static cudaError_t launch_route_d(const RouteArgs& p, cudaStream_t st) {
  const int n = p.nkb;
  if (n <= 128) return launch_route_t<D, 4, 2, 1, 8>(p, st);
  if (n <= 256) return launch_route_t<D, 8, 2, 2, 8>(p, st);
  if (n <= 384) return launch_route_t<D, 12, 2, 3, 8>(p, st);
  if (n <= 512) return launch_route_t<D, 16, 2, 4, 8>(p, st);
  if (n <= 640) return launch_route_t<D, 20, 2, 5, 8>(p, st);
  if (n <= 768) return launch_route_t<D, 24, 2, 6, 4>(p, st);
  if (n <= 1024) return launch_route_t<D, 32, 2, 8, 4>(p, st);
  if (n <= 1536) return launch_route_t<D, 48, 1, 6, 4>(p, st);
  if (n <= 2048) return launch_route_t<D, 64, 1, 8, 4>(p, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_route(const RouteArgs& p, cudaStream_t st) {
  if (p.d == 64) return launch_route_d<64>(p, st);
  if (p.d == 128) return launch_route_d<128>(p, st);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// Structured mask: one thread per (batch*head, query block). The query block's
// frames form one interval [f_lo, f_hi]; the union of their windows is
// [f_lo - window, f_hi + window]. Key block j (frames [g_lo, g_hi]) is kept when
// that interval meets [g_lo, g_hi] or when an anchor frame lies in [g_lo, g_hi].
// ---------------------------------------------------------------------------
// Adaptive window of query frame f (LVSA §2 Fenêtres Adaptatives Étendues): the local
// window [f - W, f + W] inside the video grows one frame at a time, alternately after
// and before it (a side at the edge is skipped), while |G u window| < budget.
SA_DEVI void adaptive_window(const MaskArgs& p, int f, int base, int n_valid, int& lo, int& hi) {
  const int T = p.n_frames;
  auto is_anchor = [&](int x) {
    return x >= base && x < T && (x - base) % p.period == 0 && (x - base) / p.period < p.n_anchors;
  };
  lo = max(0, f - p.window);
  hi = min(T - 1, f + p.window);
  int inside = 0;
  for (int x = lo; x <= hi; ++x) inside += is_anchor(x);
  int size = (hi - lo + 1) + n_valid - inside;
  bool after = true;
  while (size < p.budget && (lo > 0 || hi < T - 1)) {
    const int x = ((after && hi < T - 1) || lo == 0) ? ++hi : --lo;
    if (!is_anchor(x)) ++size;
    after = !after;
  }
}

__global__ void structured_mask_kernel(MaskArgs p) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (long long)p.B * p.H * p.nqb) return;
  const int i = (int)(tid % p.nqb);
  const int ft = p.frame_tokens;
  const int qs = i * p.block, qe = min(p.Nq, qs + p.block) - 1;
  const int f_lo = p.q_frame0 + qs / ft, f_hi = p.q_frame0 + qe / ft;
  const int base = p.step % p.period;
  int w_lo = f_lo - p.window, w_hi = f_hi + p.window;
  if (p.budget > 0) {
    // every frame's window contains the frame, so the union over the block's frames
    // is one interval
    int n_valid = 0;
    for (int m = 0; m < p.n_anchors && base + m * p.period < p.n_frames; ++m) ++n_valid;
    w_lo = p.n_frames;
    w_hi = -1;
    for (int f = f_lo; f <= f_hi; ++f) {
      int lo, hi;
      adaptive_window(p, f, base, n_valid, lo, hi);
      w_lo = min(w_lo, lo);
      w_hi = max(w_hi, hi);
    }
  }
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
