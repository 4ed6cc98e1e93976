// Forward pass, register-tile version: exact flash attention over the kept KV
// blocks plus order-0 / order-1 compensation of the skipped blocks, all merged in
// one online softmax.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2: Algorithme Central (o_t = N_t / D_t; exact terms for the
// kept blocks; alpha_{t,j} (sum_n v_{j,n}) for the others; the first-order term)
// and Implémentation Matérielle (phase 1 exact tiles in shared memory, phase 2 a
// sweep over the aggregated block vectors, phase 3 the first-order correction),
// with the first-order term per block: alpha_{t,j} * scale * q_t M_j.
//
// CTA: 64 query rows (4 warps x 16 rows; every CTA lies inside one query block),
// operands through a two-stage cp.async ring of 16-byte copies into swizzled
// shared memory, mma.sync m16n8k16 bf16 with fp32 accumulators in registers.
// The CTA walks one sequence of work items:
//   TILE t   64 centroids kbar_j and value sums S_j of blocks 64t..64t+63:
//            logits scale*q.kbar_j for the skipped j (kept j masked), online
//            softmax update, O += P S, l += sum_j P_j n_j
//   MAT j    (order 1, each skipped j of the current tile) U = Q M_j on the
//            tensor cores, then O += scale * P_j * U row by row
//   EXACT    64 tokens of a kept block: S = Q K^T, online softmax, O += P V
// and finally writes O / l.
#include "common.cuh"
#include "launch.h"

#include <cstdlib>
#include <type_traits>

namespace sa {

namespace fwd {

constexpr int QT = 64;        // query rows per CTA
constexpr int KT = 64;        // tokens or centroids per tile
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int MAXW = 2048 / 32;  // bitmap words (SA_MAX_KV_BLOCKS bits)
constexpr int kMaxList = 2048;   // kept-list entries held in shared memory

enum : int { kTile = 0, kMat = 1, kExact = 2, kNone = 3 };

struct Item {
  int kind, a, b;  // TILE: a = tile; MAT: a = block; EXACT: a = block, b = sub-tile
};

// Deterministic walk over the work items; every thread runs the same copy.
struct Walk {
  int phase, tile, j, p, sub;
};

template <int BLK, int ORDER>
SA_DEVI Item walk_next(Walk& w, const uint32_t* skip, const int16_t* list, int cnt, int ntiles,
                       int nkb) {
  while (true) {
    if (w.phase == 0) {
      if (w.tile >= ntiles) {
        w.phase = 1;
        continue;
      }
      if (w.j < 0) {
        w.j = w.tile * KT;
        if (skip[2 * w.tile] | skip[2 * w.tile + 1]) return Item{kTile, w.tile, 0};
        ++w.tile;
        w.j = -1;
        continue;
      }
      if (ORDER == 1) {
        const int end = min(nkb, (w.tile + 1) * KT);
        while (w.j < end) {
          const uint32_t word = skip[w.j >> 5] >> (w.j & 31);
          if (word) {
            w.j += __ffs(word) - 1;
            break;
          }
          w.j = (w.j | 31) + 1;
        }
        if (w.j < end) {
          const int jj = w.j++;
          return Item{kMat, jj, 0};
        }
      }
      ++w.tile;
      w.j = -1;
      continue;
    }
    if (w.p >= cnt) return Item{kNone, 0, 0};
    const Item it{kExact, list[w.p], w.sub};
    if (++w.sub == BLK / KT) {
      w.sub = 0;
      ++w.p;
    }
    return it;
  }
}

template <int D, int BLK, int ORDER>
struct Cfg {
  static constexpr int ROWB = D * 2;
  static constexpr int STAGE = (2 * KT * D * 2 > D * D * 2) ? 2 * KT * D * 2 : D * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = QT * ROWB;
  static constexpr int OFF_P = OFF_RING + 2 * STAGE;
  static constexpr int PSTRIDE = KT + 4;
  static constexpr int P_BYTES = ORDER == 1 ? WARPS * 16 * PSTRIDE * 4 : 0;
  static constexpr int OFF_SKIP = OFF_P + P_BYTES;
  static constexpr int OFF_LIST = OFF_SKIP + MAXW * 4;
  static constexpr int SMEM = OFF_LIST + kMaxList * 2;
};

template <int D, int BLK, int ORDER>
__global__ void __launch_bounds__(THREADS, 2)
forward_kernel(ForwardArgs p) {
  using C = Cfg<D, BLK, ORDER>;
  constexpr int ROWB = C::ROWB;
  constexpr int KSTEPS = D / 16;   // k-steps over the head dim
  constexpr int NT_O = D / 8;      // n-tiles of the output
  constexpr int NT_S = KT / 8;     // n-tiles of a logit tile
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* skip = reinterpret_cast<uint32_t*>(smem + C::OFF_SKIP);
  int16_t* list = reinterpret_cast<int16_t*>(smem + C::OFF_LIST);
  const uint32_t sbase = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int g = lane / 4, t = lane % 4;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * QT;
  const int qblk = q0 / BLK;
  const int nkb = p.nkb;
  const int ntiles = (nkb + KT - 1) / KT;
  const float sl2 = p.scale * kLog2e;   // logits in base-2 units

  const uint16_t* qg = p.q + (size_t)bh * p.Nq * D;
  const uint16_t* kg = p.k + (size_t)bh * p.Nk * D;
  const uint16_t* vg = p.v + (size_t)bh * p.Nk * D;
  const uint16_t* kbg = p.kbar16 + (size_t)bh * nkb * D;
  const uint16_t* vsg = p.vsum16 + (size_t)bh * nkb * D;
  const uint16_t* mg = ORDER == 1 ? p.M + (size_t)bh * nkb * D * D : nullptr;

  // ---- Q tile -> shared (own cp.async group) ----
  for (int x = tid; x < QT * D / 8; x += THREADS) {
    const int r = x / (D / 8), ch = x % (D / 8);
    const bool ok = q0 + r < p.Nq;
    cp_async16(sbase + C::OFF_Q + swz(r, ch, ROWB), qg + (ok ? (size_t)(q0 + r) * D + ch * 8 : 0),
               ok ? 16 : 0);
  }
  cp_async_commit();

  // ---- kept list (valid entries, order kept) and skipped-block bitmap ----
  int cnt = 0;
  {
    const size_t row = (size_t)bh * p.nqb + qblk;
    const int n_in = min(max(p.kv_cnt[row], 0), p.cap);
    const int32_t* src = p.kv_idx + row * p.cap;
    if (warp == 0) {
      for (int w = lane; w < MAXW; w += 32) skip[w] = 0u;
      __syncwarp();
      for (int base = 0; base < n_in; base += 32) {
        const int x = base + lane < n_in ? src[base + lane] : -1;
        const bool ok = x >= 0 && x < nkb;
        const unsigned bal = __ballot_sync(0xffffffffu, ok);
        if (ok) {
          const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
          if (pos < kMaxList) list[pos] = (int16_t)x;
          atomicOr(&skip[x >> 5], 1u << (x & 31));
        }
        cnt += __popc(bal);
      }
      cnt = min(cnt, kMaxList);
      __syncwarp();
      // kept bits -> skipped bits, restricted to [0, nkb)
      for (int w = lane; w < MAXW; w += 32) {
        const int lo = w * 32;
        uint32_t valid = lo + 32 <= nkb ? 0xffffffffu : (lo < nkb ? (1u << (nkb - lo)) - 1u : 0u);
        skip[w] = ~skip[w] & valid;
      }
    }
    cnt = __shfl_sync(0xffffffffu, cnt, 0);
  }
  __shared__ int s_cnt;
  if (tid == 0) s_cnt = cnt;
  cp_async_wait<0>();
  __syncthreads();
  cnt = s_cnt;

  // ---- Q fragments in registers ----
  uint32_t qf[KSTEPS][4];
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) {
    const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = kk * 16 + ((lane >> 4) & 1) * 8;
    ldsm_x4(sbase + C::OFF_Q + swz(r, col / 8, ROWB), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }

  float o[NT_O][4];
#pragma unroll
  for (int nt = 0; nt < NT_O; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY};
  float lrow[2] = {0.f, 0.f};
  float* pbuf = reinterpret_cast<float*>(smem + C::OFF_P) + warp * 16 * C::PSTRIDE;

  // ---- stage loader ----
  auto load = [&](const Item& it, int stage) {
    const uint32_t dst = sbase + C::OFF_RING + stage * C::STAGE;
    if (it.kind == kMat) {
      const uint16_t* src = mg + (size_t)it.a * D * D;
      for (int x = tid; x < D * D / 8; x += THREADS) {
        const int r = x / (D / 8), ch = x % (D / 8);
        cp_async16(dst + swz(r, ch, ROWB), src + (size_t)r * D + ch * 8, 16);
      }
      return;
    }
    const uint16_t *s0, *s1;
    int first, limit;
    if (it.kind == kTile) {
      first = it.a * KT;
      limit = nkb;
      s0 = kbg;
      s1 = vsg;
    } else {
      first = it.a * BLK + it.b * KT;
      limit = p.Nk;
      s0 = kg;
      s1 = vg;
    }
    for (int x = tid; x < KT * D / 8; x += THREADS) {
      const int r = x / (D / 8), ch = x % (D / 8);
      const bool ok = first + r < limit;
      const size_t off = ok ? (size_t)(first + r) * D + ch * 8 : 0;
      cp_async16(dst + swz(r, ch, ROWB), s0 + off, ok ? 16 : 0);
      cp_async16(dst + KT * ROWB + swz(r, ch, ROWB), s1 + off, ok ? 16 : 0);
    }
  };

  // S(16 x KT) = Q K^T for this warp's rows; keys at `kb` (KT rows, swizzled). With
  // HALF, the keys are the fp16 centroid table and Q is converted to fp16 (exact).
  auto qk = [&](uint32_t kb, float (&s)[NT_S][4], auto half_tag) {
    constexpr bool HALF = decltype(half_tag)::value;
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) a[e] = HALF ? bf16x2_to_f16x2(qf[kk][e]) : qf[kk][e];
#pragma unroll
      for (int np = 0; np < NT_S / 2; ++np) {
        const int r = np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz(r, col / 8, ROWB), b0, b1, b2, b3);
        if (HALF) {
          mma_f16(s[2 * np], a, b0, b1);
          mma_f16(s[2 * np + 1], a, b2, b3);
        } else {
          mma_bf16(s[2 * np], a, b0, b1);
          mma_bf16(s[2 * np + 1], a, b2, b3);
        }
      }
    }
  };

  // Online-softmax update with masked base-2 logits already in s; turns s into P.
  auto softmax_update = [&](float (&s)[NT_S][4]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[h], mx);
      const float corr = mnew == -INFINITY ? 1.f : exp2f(mrow[h] - mnew);
      const float mref = mnew == -INFINITY ? 0.f : mnew;
      mrow[h] = mnew;
      lrow[h] *= corr;
#pragma unroll
      for (int nt = 0; nt < NT_O; ++nt) {
        o[nt][2 * h] *= corr;
        o[nt][2 * h + 1] *= corr;
      }
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) {
        s[nt][2 * h] = exp2f(s[nt][2 * h] - mref);
        s[nt][2 * h + 1] = exp2f(s[nt][2 * h + 1] - mref);
      }
    }
  };

  // O += P(16 x KT) V(KT x D); values at `vb` (KT rows, swizzled). With HALF, P and
  // the values (the fp16 value-sum table) are fp16.
  auto pv = [&](const float (&s)[NT_S][4], uint32_t vb, auto half_tag) {
    constexpr bool HALF = decltype(half_tag)::value;
    auto pk = [&](float x, float y) { return HALF ? pack_f16(x, y) : pack_bf16(x, y); };
#pragma unroll
    for (int kk = 0; kk < KT / 16; ++kk) {
      uint32_t a[4];
      a[0] = pk(s[2 * kk][0], s[2 * kk][1]);
      a[1] = pk(s[2 * kk][2], s[2 * kk][3]);
      a[2] = pk(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      a[3] = pk(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < NT_O / 2; ++np) {
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = np * 16 + ((lane >> 4) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz(r, col / 8, ROWB), b0, b1, b2, b3);
        if (HALF) {
          mma_f16(o[2 * np], a, b0, b1);
          mma_f16(o[2 * np + 1], a, b2, b3);
        } else {
          mma_bf16(o[2 * np], a, b0, b1);
          mma_bf16(o[2 * np + 1], a, b2, b3);
        }
      }
    }
  };
  using kHalf = std::true_type;
  using kBf16 = std::false_type;

  Walk wk{0, 0, -1, 0, 0};
  Item cur = walk_next<BLK, ORDER>(wk, skip, list, cnt, ntiles, nkb);
  if (cur.kind != kNone) load(cur, 0);
  cp_async_commit();
  int stage = 0;
  int cur_tile = 0;
  while (cur.kind != kNone) {
    const Item nxt = walk_next<BLK, ORDER>(wk, skip, list, cnt, ntiles, nkb);
    if (nxt.kind != kNone) load(nxt, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sb = sbase + C::OFF_RING + stage * C::STAGE;

    if (cur.kind == kTile) {
      cur_tile = cur.a;
      float s[NT_S][4];
      qk(sb, s, kHalf{});
      float wn[NT_S][2];  // token count n_j of each column (0 where masked)
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = cur.a * KT + nt * 8 + 2 * t + e;
          const bool on = j < nkb && ((skip[j >> 5] >> (j & 31)) & 1u);
          wn[nt][e] = on ? (float)min(BLK, p.Nk - j * BLK) : 0.f;
          s[nt][e] = on ? s[nt][e] * sl2 : -INFINITY;
          s[nt][2 + e] = on ? s[nt][2 + e] * sl2 : -INFINITY;
        }
      softmax_update(s);
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) {
        lrow[0] += s[nt][0] * wn[nt][0] + s[nt][1] * wn[nt][1];
        lrow[1] += s[nt][2] * wn[nt][0] + s[nt][3] * wn[nt][1];
      }
      if (ORDER == 1) {
#pragma unroll
        for (int nt = 0; nt < NT_S; ++nt) {
          *reinterpret_cast<float2*>(pbuf + g * C::PSTRIDE + nt * 8 + 2 * t) =
              make_float2(s[nt][0], s[nt][1]);
          *reinterpret_cast<float2*>(pbuf + (g + 8) * C::PSTRIDE + nt * 8 + 2 * t) =
              make_float2(s[nt][2], s[nt][3]);
        }
      }
      pv(s, sb + KT * ROWB, kHalf{});
    } else if (cur.kind == kMat) {
      if constexpr (ORDER == 1) {
        __syncwarp();
        const int col = cur.a - cur_tile * KT;
        const float a0 = p.scale * pbuf[g * C::PSTRIDE + col];
        const float a1 = p.scale * pbuf[(g + 8) * C::PSTRIDE + col];
        float u[NT_O][4];
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) u[nt][0] = u[nt][1] = u[nt][2] = u[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          uint32_t a[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) a[e] = bf16x2_to_f16x2(qf[kk][e]);
#pragma unroll
          for (int np = 0; np < NT_O / 2; ++np) {
            const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int cc = np * 16 + ((lane >> 4) & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sb + swz(r, cc / 8, ROWB), b0, b1, b2, b3);
            mma_f16(u[2 * np], a, b0, b1);
            mma_f16(u[2 * np + 1], a, b2, b3);
          }
        }
#pragma unroll
        for (int nt = 0; nt < NT_O; ++nt) {
          o[nt][0] = fmaf(a0, u[nt][0], o[nt][0]);
          o[nt][1] = fmaf(a0, u[nt][1], o[nt][1]);
          o[nt][2] = fmaf(a1, u[nt][2], o[nt][2]);
          o[nt][3] = fmaf(a1, u[nt][3], o[nt][3]);
        }
      }
    } else {
      float s[NT_S][4];
      qk(sb, s, kBf16{});
      const int tok0 = cur.a * BLK + cur.b * KT;
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool on = tok0 + nt * 8 + 2 * t + e < p.Nk;
          s[nt][e] = on ? s[nt][e] * sl2 : -INFINITY;
          s[nt][2 + e] = on ? s[nt][2 + e] * sl2 : -INFINITY;
        }
      softmax_update(s);
#pragma unroll
      for (int nt = 0; nt < NT_S; ++nt) {
        lrow[0] += s[nt][0] + s[nt][1];
        lrow[1] += s[nt][2] + s[nt][3];
      }
      pv(s, sb + KT * ROWB, kBf16{});
    }
    __syncthreads();
    cur = nxt;
    stage ^= 1;
  }

  // ---- epilogue: O / l ----
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = lrow[h];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int row = q0 + warp * 16 + g + 8 * h;
    if (row >= p.Nq) continue;
    const size_t base = ((size_t)bh * p.Nq + row) * D;
#pragma unroll
    for (int nt = 0; nt < NT_O; ++nt) {
      const float x0 = o[nt][2 * h] * inv, x1 = o[nt][2 * h + 1] * inv;
      const int c = nt * 8 + 2 * t;
      if (p.out_dtype == 0) {
        *reinterpret_cast<float2*>(static_cast<float*>(p.out) + base + c) = make_float2(x0, x1);
      } else {
        *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + base + c) = pack_bf16(x0, x1);
      }
    }
  }
}

}  // namespace fwd

template <int D, int BLK, int ORDER>
static cudaError_t launch_forward_t(const ForwardArgs& p, cudaStream_t st) {
  using C = fwd::Cfg<D, BLK, ORDER>;
  auto kern = fwd::forward_kernel<D, BLK, ORDER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((p.Nq + fwd::QT - 1) / fwd::QT, p.B * p.H);
  kern<<<grid, fwd::THREADS, C::SMEM, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_forward_mma(const ForwardArgs& p, cudaStream_t st) {
#define SA_FWD_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && p.order == O_) return launch_forward_t<D_, B_, O_>(p, st);
  SA_FWD_CASE(64, 64, 0) SA_FWD_CASE(64, 64, 1) SA_FWD_CASE(64, 128, 0) SA_FWD_CASE(64, 128, 1)
  SA_FWD_CASE(128, 64, 0) SA_FWD_CASE(128, 64, 1) SA_FWD_CASE(128, 128, 0) SA_FWD_CASE(128, 128, 1)
#undef SA_FWD_CASE
  return cudaErrorInvalidValue;
}

// The tcgen05 kernel is the forward; the register-tile kernel stays selectable with
// SPARSE_ATTN_FORWARD=mma for side-by-side measurements.
cudaError_t launch_forward(const ForwardArgs& p, cudaStream_t st) {
  static const int use_mma = [] {
    const char* e = getenv("SPARSE_ATTN_FORWARD");
    return e && e[0] == 'm' ? 1 : 0;
  }();
  return use_mma ? launch_forward_mma(p, st) : launch_forward_tc(p, st);
}

}  // namespace sa
