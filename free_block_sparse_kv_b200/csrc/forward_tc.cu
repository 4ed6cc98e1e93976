// Forward pass on the 5th-generation tensor cores: tcgen05.mma with accumulators in
// tensor memory, operands staged by TMA, one warp-specialised CTA per 128 query rows.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2: Algorithme Central (o_t = N_t / D_t; exact terms for the kept
// blocks; alpha_{t,j} (sum_n v_{j,n}) for the others; the first-order term, here per
// block: alpha_{t,j} * scale * q_t M_j) and Implémentation Matérielle (phase 1 exact
// tiles in on-chip memory, phase 2 a sweep over the aggregated block vectors, phase 3
// the first-order correction), all merged into one online softmax.
//
// Roles (384 threads):
//   warps 0-7  softmax. Warps w and w+4 share TMEM lanes 32*(w%4).. (query rows) and
//              split each row's columns in halves; they exchange row maxima and row
//              sums through shared memory. They read logits from TMEM, keep the running
//              max (rescaling O lazily, only when a row's max grows by more than 2^11),
//              write P back to TMEM as the A operand of the value product, and build the
//              order-1 operand A_j = (scale * alpha_tj) q_t in TMEM.
//   warp 8     TMA producer: Q once, then every operand tile through a 5 x 32 KB ring.
//   warp 9     allocates TMEM; lane 0 issues every tcgen05.mma and commit.
//   warps 10-11 idle (they complete the control warpgroup for the register split).
// Work items, in order (the same walk runs in all three roles):
//   TILE t   64 centroids (bf16 hi + lo) and value sums (fp16):
//            S = Q Kbar_hi^T + Q Kbar_lo^T, P, O += P S
//   MAT j    each pair of skipped blocks of the current tile (order 1):
//            O += [A_j1 | A_j2] [M_j1; M_j2] (fp16)
//   EXACT j  each kept block: S = Q K_j^T (bf16), P, O += P V_j (fp16 P and V)
// The MMA warp issues the logits of the next TILE/EXACT item before the value
// product of the current one, so logits overlap the softmax of the previous item.
// TMEM columns: O [0, D); S/P buffers R0 = [128, 256), R1 = [256, 384); A slot 0 at
// [384, 512). Order-1 products go two skipped blocks at a time: A = [a1 q | a2 q]
// (K = 2d) against [M_j1; M_j2], 16 tensor-core instructions per hand-off. During a
// tile's MAT items the tile's S/P buffer is free once its value product has run (the
// tile's P is also kept in shared memory for alpha) and serves as A slot 1.
// Every mbarrier wait is bounded: on timeout the CTA sets err_flag, abandons its work,
// drains its own TMA loads and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace sa {
namespace tcf {

constexpr int TQ = 128;        // query rows per CTA
constexpr int KC = 64;         // centroids per TILE item
constexpr int NU = 5;          // ring units
constexpr int UNIT = 32768;    // bytes per ring unit
constexpr int MAXW = 64;       // bitmap words (2048 blocks)
constexpr int NSOFT = 256;     // softmax threads (8 warps, 2 warpgroups)
constexpr int NTHREADS = NSOFT + 128;  // + one control warpgroup (producer, MMA, 2 idle)
// Register split after launch (168 per thread at launch = 64,512 per CTA): the
// control warpgroup gives registers back, the softmax warpgroups take them.
constexpr int kRegCtl = 72, kRegSoft = 208;
static_assert(2 * 128 * kRegSoft + 128 * kRegCtl <= 168 * NTHREADS, "register split");
constexpr int NA = 3;          // A-operand slots for the order-1 products (each holds a pair)
constexpr float kThresh = 11.0f;  // lazy-rescale threshold, base-2 units (P < 2^11)
constexpr uint32_t kWaitLimit = 1u << 18;  // ~0.3 s: far above any legitimate wait

constexpr uint32_t COL_O = 0, COL_R0 = 128, COL_A0 = 384;

// shared-memory map (offsets from a 1024-aligned base)
constexpr int OFF_Q = 0;                       // Q tile, bf16, swizzled (32 KB)
constexpr int OFF_U = 32768;                   // ring
constexpr int OFF_CTL = OFF_U + NU * UNIT;     // control block (2 KB)
constexpr int OFF_STASH = OFF_CTL + 2048;      // P of the current tile, fp16 [KC][TQ]
constexpr int OFF_RED = OFF_STASH + KC * TQ * 2;  // row max (2 x 2 x TQ) and sum (2 x TQ), f32
constexpr int SMEM_BYTES = OFF_RED + 6 * TQ * 4 + 1024;

struct Params {
  CUtensorMap tmQ, tmK, tmV, tmKb, tmVs, tmM;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  void* out;
  int32_t* err_flag;
  int cap, Nq, Nk, nqb, nkb, out_dtype;
  float scale;
};

struct Ctl {  // control block in shared memory
  uint64_t full[NU], empty[NU];
  uint64_t s_full[2], p_full[2], pv_done[2], s_free[2];
  uint64_t a_full[NA], a_done[NA];
  uint64_t q_full, init_done, drain;
  uint64_t pair[4];         // the two softmax warps sharing 32 rows
  int4 evq[NU];             // event of each ring unit: {kind | item kind << 4, j, buf | tbuf << 4, use}
  uint32_t tmem_base;
  int abort;
  uint32_t kept[2][MAXW];   // kept blocks of each query block in the tile (half)
  uint32_t keptU[MAXW];     // union: EXACT items
  uint32_t skipU[MAXW];     // union of skipped blocks: TILE / MAT items
};
static_assert(sizeof(Ctl) <= 2048, "control block");

enum : int { kTile = 0, kMat = 1, kExact = 2, kNone = 3 };
struct Item {
  int kind, j;  // TILE: j = tile index; MAT / EXACT: j = block index
  int j2 = -1;  // MAT: second skipped block of the pair, or -1
};

// The walk over work items; identical in every role. The skipped blocks of the
// current tile and the kept blocks of the current 32-block word are held in
// registers as bit masks, so each step is a few integer instructions.
struct Walk {
  int phase = 0, tile = 0, word = 0;
  uint64_t tmask = 0;  // phase 0: skipped blocks of `tile` not yet walked
  uint32_t kmask = 0;  // phase 1: kept blocks of `word` not yet walked
  bool in_tile = false;
  template <int ORDER>
  SA_DEVI Item next(const Ctl& c, int nkb) {
    const int ntiles = (nkb + KC - 1) / KC;
    while (true) {
      if (phase == 0) {
        if (!in_tile) {
          if (tile >= ntiles) {
            phase = 1;
            word = 0;
            kmask = c.keptU[0];
            continue;
          }
          tmask = (uint64_t)c.skipU[2 * tile] | ((uint64_t)c.skipU[2 * tile + 1] << 32);
          if (tmask) {
            in_tile = true;
            return Item{kTile, tile};
          }
          ++tile;
          continue;
        }
        if (ORDER == 1 && tmask) {
          // skipped blocks of this tile, two at a time
          const int j1 = tile * KC + __ffsll((long long)tmask) - 1;
          tmask &= tmask - 1;
          int j2 = -1;
          if (tmask) {
            j2 = tile * KC + __ffsll((long long)tmask) - 1;
            tmask &= tmask - 1;
          }
          return Item{kMat, j1, j2};
        }
        in_tile = false;
        ++tile;
        continue;
      }
      while (!kmask) {
        if (++word >= (nkb + 31) / 32) return Item{kNone, 0};
        kmask = c.keptU[word];
      }
      const int j = word * 32 + __ffs(kmask) - 1;
      kmask &= kmask - 1;
      return Item{kExact, j};
    }
  }
};

// MMA-side event stream. The logits of the next TILE/EXACT item are issued before
// the value product of the current one (look-ahead), except after an order-1 TILE:
// there they follow the tile's order-1 products, which use the other S/P buffer.
enum : int { eS = 0, ePV = 1, eMat = 2, eNone = 3 };
struct Event {
  int kind;   // eS, ePV, eMat, eNone
  Item item;
  int buf, use;   // S / PV: S-buffer and its use count; MAT: A slot and its use count
  int tbuf;       // MAT: S-buffer of the tile the block belongs to
};
struct EventGen {
  Walk cur, ahead;
  int ns_ahead = 0, ns_cur = 0, nmat = 0, tile_buf = 0;
  bool started = false;
  Event q0, q1;  // queued events (at most two)
  int nq = 0;

  template <int ORDER>
  SA_DEVI Item next_s(const Ctl& c, int nkb) {
    while (true) {
      Item it = ahead.template next<ORDER>(c, nkb);
      if (it.kind != kMat) return it;
    }
  }
  template <int ORDER>
  SA_DEVI Event next(const Ctl& c, int nkb) {
    if (nq) {
      const Event e = q0;
      q0 = q1;
      --nq;
      return e;
    }
    if (!started) {
      started = true;
      Item s = next_s<ORDER>(c, nkb);
      if (s.kind == kNone) return Event{eNone, s, 0, 0, 0};
      const int n = ns_ahead++;
      return Event{eS, s, n & 1, n >> 1, 0};
    }
    Item it = cur.template next<ORDER>(c, nkb);
    if (it.kind == kNone) return Event{eNone, it, 0, 0, 0};
    if (it.kind == kMat) {
      const int n = nmat++;
      return Event{eMat, it, n % NA, n / NA, tile_buf};
    }
    const int n = ns_cur++;
    if (it.kind == kTile) tile_buf = n & 1;
    const Event pv{ePV, it, n & 1, n >> 1, 0};
    Event first = pv;
    bool have_first = false;
    if (ns_ahead <= n) {  // this item's logits were deferred
      const Item s = next_s<ORDER>(c, nkb);
      const int m = ns_ahead++;
      first = Event{eS, s, m & 1, m >> 1, 0};
      have_first = true;
    }
    if (!(ORDER == 1 && it.kind == kTile)) {
      const Item s = next_s<ORDER>(c, nkb);
      if (s.kind != kNone) {
        const int m = ns_ahead++;
        const Event la{eS, s, m & 1, m >> 1, 0};
        if (have_first) {
          q0 = la;
          nq = 1;
        } else {
          first = la;
          have_first = true;
        }
      }
    }
    if (have_first) {
      if (nq == 0) q0 = pv; else q1 = pv;
      ++nq;
    }
    return first;
  }
};

// TMEM column of A slot `slot` (128 columns: the operands of two skipped blocks) for a
// tile whose S/P buffer is `tbuf`. Slot 1 reuses that buffer once its P has been read;
// slot 2 is the other S/P buffer, left free during a tile's order-1 products (the
// logits of the next item are issued after them).
SA_DEVI uint32_t a_col(int slot, int tbuf) {
  return slot == 0 ? COL_A0 : COL_R0 + 128 * (slot == 1 ? tbuf : 1 - tbuf);
}

template <int D, int BLK>
struct Bytes {
  static constexpr int SUB = D / 64;                    // 64-column sub-tiles per row
  static constexpr uint32_t KB = SUB * KC * 128;        // centroid tile
  static constexpr uint32_t VS = SUB * KC * 128;        // value-sum tile
  static constexpr uint32_t M = SUB * D * 128;          // one M_j
  static constexpr uint32_t KV = SUB * BLK * 128;       // one K or V block
  static constexpr uint32_t Q = SUB * TQ * 128;         // query tile
};

// TMEM store of W consecutive 32-bit columns (W = 16 or 32).
template <int W>
SA_DEVI void tmem_st_w(uint32_t taddr, const uint32_t* r) {
  if constexpr (W == 32) {
    tc::tmem_st32(taddr, r);
  } else {
    static_assert(W == 16, "width");
    tc::tmem_st16(taddr, r);
  }
}

// Softmax warps. Thread (warp w, lane l) owns query row r = 32*(w%4) + l and the
// column half w/4 of every logit tile; the two threads of a row meet through an
// mbarrier of their warp pair (bounded waits, so an abort never strands a partner).
template <int D, int BLK, int ORDER>
SA_DEVI void softmax_role(const Params& p, Ctl& c, uint8_t* gbase, uint32_t tmem, tc::Waiter& wt,
                          int warp, int lane) {
  constexpr int SUB = D / 64;
  constexpr int DH = D / 2;  // O columns per thread
  constexpr int AW = D / 4;  // A-operand columns (fp16 pairs) per thread
  const int qw = warp & 3, ch = warp >> 2;
  const int r = 32 * qw + lane;
  const uint32_t lane_off = (uint32_t)(32 * qw) << 16;
  const int h = BLK == 64 ? (r >> 6) : 0;  // which query block of the tile
  const float sl2 = p.scale * kLog2e;
  const int nkb = p.nkb;
  const int bh = blockIdx.y, q0 = blockIdx.x * TQ;
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };
  auto uni = [](bool x) { return __all_sync(0xffffffffu, x); };
  float* red = reinterpret_cast<float*>(gbase + OFF_RED);       // max [2][2][TQ], sum [2][TQ]
  __half* stash = reinterpret_cast<__half*>(gbase + OFF_STASH);  // [KC][TQ]
  // One arrival per warp: every lane's tensor-memory stores are ordered before the
  // warp barrier, and lane 0 arrives after it.
  auto warp_arrive = [&](uint32_t b) {
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(b);
  };
  const uint32_t pbar = bar(c.pair[qw]);
  int pair_phase = 0;
  auto pair_sync = [&]() {
    warp_arrive(pbar);
    const bool r2 = uni(wt.fast(pbar, pair_phase & 1, 14));
    ++pair_phase;
    return r2;
  };

  bool ok = uni(wt.wait(bar(c.q_full), 0, 9));
  // fp16 copy of this thread's half of its Q row, in registers (order-1 operands)
  uint32_t q16[AW];
#pragma unroll
  for (int i = 0; i < 4 * SUB; ++i) {
    const int cc = ch * 4 * SUB + i;
    const int s = cc / 8, cw = cc % 8;
    const uint32_t off = s * TQ * 128 + r * 128 + ((cw ^ (r & 7)) << 4);
    const uint4 x = *reinterpret_cast<const uint4*>(gbase + OFF_Q + off);
    const uint4 y = make_uint4(bf16x2_to_f16x2(x.x), bf16x2_to_f16x2(x.y), bf16x2_to_f16x2(x.z),
                               bf16x2_to_f16x2(x.w));
    q16[4 * i + 0] = y.x;
    q16[4 * i + 1] = y.y;
    q16[4 * i + 2] = y.z;
    q16[4 * i + 3] = y.w;
  }
  tc::fence_proxy_async();
  {
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
    for (int k = 0; k < DH / 32; ++k) tc::tmem_st32(tmem + lane_off + COL_O + ch * DH + 32 * k, z);
    tc::tmem_wait_st();
  }
  warp_arrive(bar(c.init_done));

  float m_ref = -INFINITY, l = 0.f;
  // The last O-writing MMA issued before our next value product: kind 0 = value
  // product of S-buffer lw_buf, kind 1 = order-1 product of A slot lw_buf.
  int lw_kind = -1, lw_buf = 0, lw_use = 0;
  auto wait_last_writer = [&](int where) {
    if (lw_kind < 0) return true;
    const uint32_t b = lw_kind == 0 ? bar(c.pv_done[lw_buf]) : bar(c.a_done[lw_buf]);
    const bool r2 = uni(wt.wait(b, lw_use & 1, where));
    tc::fence_after_sync();
    return r2;
  };

  Walk wk;
  int ns = 0, nmat = 0, cur_buf = 0, cur_use = 0, cur_tile = 0, prev_buf = -1;
  bool r_slots_free = false;  // this tile's value product has read its P

  // One TILE (IS_TILE, NH = 32) or EXACT (NH = BLK / 2) item: this thread's NH logits.
  auto s_item = [&](const Item& it, int sb, int n, auto nh_tag, auto tile_tag) -> bool {
    constexpr int NH = decltype(nh_tag)::value;
    constexpr bool TILE = decltype(tile_tag)::value;
    constexpr int NK = NH / 32;
    const uint32_t sa = tmem + lane_off + COL_R0 + 128 * sb;
    const int col0 = ch * NH;
    uint32_t sv[NH];
#pragma unroll
    for (int k = 0; k < NK; ++k)
      tc::tmem_ld32(sa + col0 + 32 * k, sv + 32 * k);
    tc::tmem_wait_ld();
    uint32_t mbits[NK];
#pragma unroll
    for (int k = 0; k < NK; ++k) {
      if (TILE) {
        const int j0 = it.j * KC + col0 + 32 * k;
        mbits[k] = c.skipU[j0 >> 5] & ~c.kept[h][j0 >> 5];
      } else {
        const int t0 = it.j * BLK + col0 + 32 * k;
        mbits[k] = t0 + 32 <= p.Nk ? 0xffffffffu : (t0 < p.Nk ? (1u << (p.Nk - t0)) - 1u : 0u);
        if (BLK == 64 && !((c.kept[h][it.j >> 5] >> (it.j & 31)) & 1u)) mbits[k] = 0u;
      }
    }
    // Logits in base-2 units; masked columns become -inf, which the exponential maps
    // to an exact zero, so the second pass needs no per-column tests.
    float xv[NH];
#pragma unroll
    for (int k = 0; k < NK; ++k)
#pragma unroll
      for (int i = 0; i < 32; ++i)
        xv[32 * k + i] = ((mbits[k] >> i) & 1u) ? __uint_as_float(sv[32 * k + i]) * sl2 : -INFINITY;
    float mx;
    {
      float m8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) m8[a] = xv[a];
#pragma unroll
      for (int i = 8; i < NH; ++i) m8[i % 8] = fmaxf(m8[i % 8], xv[i]);
      mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    }
    float* rmax = red + (n & 1) * 2 * TQ;
    rmax[ch * TQ + r] = mx;
    if (!pair_sync()) return false;
    mx = fmaxf(mx, rmax[(1 - ch) * TQ + r]);
    // Lazy rescale: only rows whose max grew by more than 2^kThresh move their
    // reference; rows that had no reference yet just take one (O is still zero).
    const bool grow = mx > m_ref + kThresh;
    const bool need_o = grow && m_ref != -INFINITY;
    const float f = need_o ? tc::ex2(m_ref - mx) : 1.f;
    if (grow) m_ref = mx;
    l *= f;
    if (__any_sync(0xffffffffu, need_o)) {
      if (!wait_last_writer(12)) return false;
#pragma unroll
      for (int k = 0; k < DH / 32; ++k) {
        uint32_t v[32];
        const uint32_t oa = tmem + lane_off + COL_O + ch * DH + 32 * k;
        tc::tmem_ld32(oa, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
        tc::tmem_st32(oa, v);
      }
      tc::tmem_wait_st();
    }
    // P = 2^(x - m_ref) as fp16 pairs over the logits of both halves (all of them were
    // read before the pair met, so the writes cannot overtake a partner's read).
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
    // TILE: column of the possibly partial last block within this half, and its P
    const int jl = TILE ? nkb - 1 - (it.j * KC + col0) : -1;
    float plast = 0.f;
#pragma unroll
    for (int k = 0; k < NK; ++k) {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float x0 = tc::ex2(xv[32 * k + i] - m_ref);
        const float x1 = tc::ex2(xv[32 * k + i + 1] - m_ref);
        l4[(i / 2) & 3] += x0 + x1;
        pk[i / 2] = pack_f16(x0, x1);
        if (TILE) {
          stash[(col0 + 32 * k + i) * TQ + r] = __float2half_rn(x0);
          stash[(col0 + 32 * k + i + 1) * TQ + r] = __float2half_rn(x1);
          plast = (32 * k + i == jl) ? x0 : ((32 * k + i + 1 == jl) ? x1 : plast);
        }
      }
      tc::tmem_st16(sa + col0 / 2 + 16 * k, pk);
    }
    if (TILE) {
      // order-0 denominator weight n_j: b for every block but a partial last one
      float lt = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      lt *= (float)BLK;
      lt += plast * (float)(p.Nk - nkb * BLK);
      l += lt;
    } else {
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
    }
    tc::tmem_wait_st();
    warp_arrive(bar(c.p_full[sb]));
    if (TILE && !pair_sync()) return false;  // the partner's half of the stash is visible
    return true;
  };

  while (ok) {
    const Item it = wk.next<ORDER>(c, nkb);
    if (it.kind == kNone) break;
    if (it.kind == kMat) {
      if constexpr (ORDER == 1) {
        const int n = nmat++;
        const int slot = n % NA, use = n / NA;
        if (use >= 1) ok = uni(wt.fast(bar(c.a_done[slot]), (use - 1) & 1, 10));
        if (ok && slot == 1 && !r_slots_free) {
          ok = uni(wt.wait(bar(c.pv_done[cur_buf]), cur_use & 1, 15));
          r_slots_free = true;
        }
        if (!ok) break;
        tc::fence_after_sync();
        const uint32_t ab = tmem + lane_off + a_col(slot, cur_buf) + ch * AW;
        const int jb[2] = {it.j, it.j2};
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (jb[b] < 0) break;
          const float pj = __half2float(stash[(jb[b] - cur_tile * KC) * TQ + r]);
          const __half2 al = __float2half2_rn(pj * p.scale);
          uint32_t a[AW];
#pragma unroll
          for (int i = 0; i < AW; ++i) {
            const __half2 y = __hmul2(*reinterpret_cast<const __half2*>(&q16[i]), al);
            a[i] = *reinterpret_cast<const uint32_t*>(&y);
          }
          tmem_st_w<AW>(ab + b * (D / 2), a);
        }
        tc::tmem_wait_st();
        warp_arrive(bar(c.a_full[slot]));
        lw_kind = 1;
        lw_buf = slot;
        lw_use = use;
      }
      continue;
    }
    // ---- TILE or EXACT: logits in an S buffer ----
    if (prev_buf >= 0) warp_arrive(bar(c.s_free[prev_buf]));
    const int n = ns++;
    const int sb = n & 1, use = n >> 1;
    prev_buf = sb;
    ok = uni(wt.fast(bar(c.s_full[sb]), use & 1, 11));
    if (!ok) break;
    tc::fence_after_sync();
    if (it.kind == kTile) {
      cur_buf = sb;
      cur_use = use;
      cur_tile = it.j;
      r_slots_free = false;
      ok = s_item(it, sb, n, std::integral_constant<int, KC / 2>{}, std::true_type{});
    } else {
      ok = s_item(it, sb, n, std::integral_constant<int, BLK / 2>{}, std::false_type{});
    }
    lw_kind = 0;
    lw_buf = sb;
    lw_use = use;
  }

  // ---- epilogue: O / l over both column halves ----
  if (ok) ok = wait_last_writer(13);
  float* rsum = red + 4 * TQ;
  rsum[ch * TQ + r] = l;
  if (ok) ok = pair_sync();
  if (!ok) return;
  const float lt = l + rsum[(1 - ch) * TQ + r];
  const bool store = q0 + r < p.Nq;
  const float inv = lt > 0.f ? 1.f / lt : 0.f;
  const size_t rowoff = ((size_t)bh * p.Nq + q0 + (store ? r : 0)) * D + ch * DH;
#pragma unroll
  for (int k = 0; k < DH / 32; ++k) {
    uint32_t v[32];
    tc::tmem_ld32(tmem + lane_off + COL_O + ch * DH + 32 * k, v);
    tc::tmem_wait_ld();
    if (!store) continue;
    if (p.out_dtype == 0) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + rowoff + 32 * k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                           __uint_as_float(v[4 * i + 2]) * inv, __uint_as_float(v[4 * i + 3]) * inv);
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + rowoff + 32 * k);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = make_uint4(pack_bf16(__uint_as_float(v[8 * i + 0]) * inv, __uint_as_float(v[8 * i + 1]) * inv),
                          pack_bf16(__uint_as_float(v[8 * i + 2]) * inv, __uint_as_float(v[8 * i + 3]) * inv),
                          pack_bf16(__uint_as_float(v[8 * i + 4]) * inv, __uint_as_float(v[8 * i + 5]) * inv),
                          pack_bf16(__uint_as_float(v[8 * i + 6]) * inv, __uint_as_float(v[8 * i + 7]) * inv));
    }
  }
}

template <int D, int BLK, int ORDER>
__global__ void __launch_bounds__(NTHREADS, 1) forward_tc_kernel(const __grid_constant__ Params p) {
  using By = Bytes<D, BLK>;
  constexpr int SUB = By::SUB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  Ctl& c = *reinterpret_cast<Ctl*>(gbase + OFF_CTL);
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * TQ;
  const int nkb = p.nkb;

  // A failure reported by an earlier CTA (or call) makes the rest of the grid skip
  // its work, so a fault costs one wave, not the whole grid.
  if (tid == 0) c.abort = (p.err_flag && *reinterpret_cast<volatile int32_t*>(p.err_flag)) ? 1 : 0;
  __syncthreads();
  if (c.abort) return;

  // ---- setup: barriers (producer warp), TMEM (MMA warp), kept bitmaps (softmax) ----
  if (warp == 8 && lane == 0) {
    for (int u = 0; u < NU; ++u) {
      tc::mbar_init(bar(c.full[u]), 1);
      tc::mbar_init(bar(c.empty[u]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(bar(c.s_full[b]), 1);
      tc::mbar_init(bar(c.pv_done[b]), 1);
      tc::mbar_init(bar(c.p_full[b]), NSOFT / 32);
      tc::mbar_init(bar(c.s_free[b]), NSOFT / 32);
    }
    for (int a = 0; a < NA; ++a) {
      tc::mbar_init(bar(c.a_done[a]), 1);
      tc::mbar_init(bar(c.a_full[a]), NSOFT / 32);
    }
    tc::mbar_init(bar(c.q_full), 1);
    tc::mbar_init(bar(c.init_done), NSOFT / 32);
    tc::mbar_init(bar(c.drain), 1);
    for (int w = 0; w < 4; ++w) tc::mbar_init(bar(c.pair[w]), 2);
    tc::fence_mbar_init();
    tc::fence_proxy_async();
  }
  if (warp == 9) {
    tc::tmem_alloc(smem_u32(&c.tmem_base), 512);
    tc::tmem_relinquish();
  }
  if (warp < 8) {
    // Kept bitmaps of the one (block 128) or two (block 64) query blocks of the tile.
    const int nh = BLK == 128 ? 1 : 2;
    for (int w = tid; w < 2 * MAXW; w += NSOFT) (&c.kept[0][0])[w] = 0u;
    asm volatile("bar.sync 1, %0;\n" ::"n"(NSOFT) : "memory");
    for (int h = 0; h < nh; ++h) {
      const int qb = q0 / BLK + h;
      if (qb >= p.nqb) continue;
      const size_t row = (size_t)bh * p.nqb + qb;
      const int n = min(max(p.kv_cnt[row], 0), p.cap);
      const int32_t* src = p.kv_idx + row * p.cap;
      for (int x = tid; x < n; x += NSOFT) {
        const int j = src[x];
        if (j >= 0 && j < nkb) atomicOr(&c.kept[h][j >> 5], 1u << (j & 31));
      }
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(NSOFT) : "memory");
    const bool has1 = BLK == 64 && (q0 / BLK + 1) < p.nqb;
    for (int w = tid; w < MAXW; w += NSOFT) {
      const int lo = w * 32;
      const uint32_t valid = lo + 32 <= nkb ? 0xffffffffu : (lo < nkb ? (1u << (nkb - lo)) - 1u : 0u);
      const uint32_t k0 = c.kept[0][w];
      const uint32_t k1 = BLK == 128 ? k0 : (has1 ? c.kept[1][w] : k0);
      if (BLK == 128 || !has1) c.kept[1][w] = k0;
      c.keptU[w] = (k0 | k1) & valid;
      c.skipU[w] = (~k0 | ~k1) & valid;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  tc::Waiter wt{&c.abort, p.err_flag, kWaitLimit};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegSoft));
    softmax_role<D, BLK, ORDER>(p, c, gbase, tmem, wt, warp, lane);
  } else {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegCtl));
  if (warp == 8) {
    // =========================== TMA producer ===========================
    if (lane == 0) {
      tc::prefetch_tmap(&p.tmQ);
      tc::mbar_arrive_expect_tx(bar(c.q_full), By::Q);
      for (int s = 0; s < SUB; ++s)
        tc::tma_load_3d(base + OFF_Q + s * TQ * 128, &p.tmQ, bar(c.q_full), 64 * s, q0, bh);
      EventGen gen;
      int u = 0;
      bool ok = true;
      while (ok) {
        const Event e = gen.next<ORDER>(c, nkb);
        const int slot = u % NU;
        if (u >= NU) ok = wt.fast(bar(c.empty[slot]), ((u / NU) - 1) & 1, 1);
        if (!ok) break;
        const uint32_t dst = base + OFF_U + slot * UNIT;
        const uint32_t fb = bar(c.full[slot]);
        const Item& it = e.item;
        // The MMA thread reads the event of a unit after the unit's full barrier.
        c.evq[slot] = make_int4(e.kind | (it.kind << 4) | ((it.j2 >= 0) << 8), it.j,
                                e.buf | (e.tbuf << 4), e.use);
        if (e.kind == eNone) {
          tc::mbar_arrive(fb);  // terminal record, no data
          ++u;
          break;
        }
        if (e.kind == eS && it.kind == kTile) {
          tc::mbar_arrive_expect_tx(fb, 2 * By::KB);
          for (int pl = 0; pl < 2; ++pl)
            for (int s = 0; s < SUB; ++s)
              tc::tma_load_3d(dst + pl * By::KB + s * KC * 128, &p.tmKb, fb, 64 * s, it.j * KC,
                              2 * bh + pl);
        } else if (e.kind == ePV && it.kind == kTile) {
          tc::mbar_arrive_expect_tx(fb, By::VS);
          for (int s = 0; s < SUB; ++s)
            tc::tma_load_3d(dst + s * KC * 128, &p.tmVs, fb, 64 * s, it.j * KC, bh);
        } else if (e.kind == eMat) {
          tc::mbar_arrive_expect_tx(fb, By::M);
          for (int s = 0; s < SUB; ++s)
            tc::tma_load_3d(dst + s * D * 128, &p.tmM, fb, 64 * s, 0, bh * nkb + it.j);
          if (it.j2 >= 0) {  // the pair's second block goes to the next unit
            ++u;
            const int s2 = u % NU;
            if (u >= NU) ok = wt.fast(bar(c.empty[s2]), ((u / NU) - 1) & 1, 1);
            if (!ok) break;
            const uint32_t fb2 = bar(c.full[s2]);
            tc::mbar_arrive_expect_tx(fb2, By::M);
            for (int s = 0; s < SUB; ++s)
              tc::tma_load_3d(base + OFF_U + s2 * UNIT + s * D * 128, &p.tmM, fb2, 64 * s, 0,
                              bh * nkb + it.j2);
          }
        } else {
          const CUtensorMap* m = e.kind == eS ? &p.tmK : &p.tmV;
          tc::mbar_arrive_expect_tx(fb, By::KV);
          for (int s = 0; s < SUB; ++s)
            tc::tma_load_3d(dst + s * BLK * 128, m, fb, 64 * s, it.j * BLK, bh);
        }
        ++u;
      }
      // Drain: every load issued must land before the CTA exits.
      tc::wait_drain(bar(c.q_full), 0, kWaitLimit);
      for (int v = max(0, u - NU); v < u; ++v)
        tc::wait_drain(bar(c.full[v % NU]), (v / NU) & 1, kWaitLimit);
    }
  } else if (warp == 9) {
    // =========================== MMA issuer ===========================
    if (lane == 0) {
      constexpr uint32_t I_S_TILE = tc::idesc_f16(1, 1, 0, KC);
      constexpr uint32_t I_PV_TILE = tc::idesc_f16(0, 0, 1, D);
      constexpr uint32_t I_S_EX = tc::idesc_f16(1, 1, 0, BLK);
      constexpr uint32_t I_PV_EX = tc::idesc_f16(0, 0, 1, D);
      constexpr uint32_t I_MAT = tc::idesc_f16(0, 0, 1, D);
      bool ok = wt.wait(bar(c.init_done), 0, 2) && wt.wait(bar(c.q_full), 0, 3);
      tc::fence_after_sync();
      // Descriptor bases; per k-step only the start-address field (low bits) moves.
      const uint64_t dQ = tc::sdesc(base + OFF_Q, 16, 1024);
      for (int u = 0; ok; ++u) {
        const int slot = u % NU;
        ok = wt.fast(bar(c.full[slot]), (u / NU) & 1, 4);
        if (!ok) break;
        const int4 rec = c.evq[slot];  // ordered by the full-barrier wait (asm with memory clobber)
        const int kind = rec.x & 15, ikind = (rec.x >> 4) & 15, buf = rec.z & 15, tbuf = rec.z >> 4;
        const bool pair = (rec.x >> 8) & 1;
        const int use = rec.w;
        if (kind == eNone) break;
        const uint32_t src = base + OFF_U + slot * UNIT;
        if (kind == eS) {
          if (use >= 1) ok = wt.fast(bar(c.s_free[buf]), (use - 1) & 1, 5);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t dt = tmem + COL_R0 + 128 * buf;
          const bool tile = ikind == kTile;
          const int rows = tile ? KC : BLK;
          const uint64_t bd0 = tc::sdesc(src, 16, 1024);
          const uint32_t idesc = tile ? I_S_TILE : I_S_EX;
          // tile: the hi plane, then the lo plane of the centroids, into the same logits
          const int planes = tile ? 2 : 1;
          for (int pl = 0; pl < planes; ++pl)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t aoff = ((kk / 4) * TQ * 128 + (kk % 4) * 32) >> 4;
              const uint32_t boff = (pl * By::KB + (kk / 4) * rows * 128 + (kk % 4) * 32) >> 4;
              tc::mma_ss(dt, dQ + aoff, bd0 + boff, idesc, (pl | kk) > 0);
            }
          tc::mma_commit(bar(c.s_full[buf]));
        } else if (kind == ePV) {
          ok = wt.fast(bar(c.p_full[buf]), use & 1, 6);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t pa = tmem + COL_R0 + 128 * buf;
          const bool tile = ikind == kTile;
          const int rows = tile ? KC : BLK;
          const uint64_t bd0 = tc::sdesc(src, rows * 128, 1024);
          const uint32_t idesc = tile ? I_PV_TILE : I_PV_EX;
          for (int kk = 0; kk < rows / 16; ++kk)
            tc::mma_ts(tmem + COL_O, pa + kk * 8, bd0 + ((kk * 2048) >> 4), idesc, 1);
          tc::mma_commit(bar(c.pv_done[buf]));
        } else {
          const int slot2 = (u + 1) % NU;
          if (pair) ok = wt.fast(bar(c.full[slot2]), ((u + 1) / NU) & 1, 4);
          if (ok) ok = wt.fast(bar(c.a_full[buf]), use & 1, 7);
          if (!ok) break;
          tc::fence_after_sync();
          const uint32_t aa = tmem + a_col(buf, tbuf);
          const uint64_t bd0 = tc::sdesc(src, D * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tc::mma_ts(tmem + COL_O, aa + kk * 8, bd0 + ((kk * 2048) >> 4), I_MAT, 1);
          if (pair) {
            const uint64_t bd1 = tc::sdesc(base + OFF_U + slot2 * UNIT, D * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              tc::mma_ts(tmem + COL_O, aa + D / 2 + kk * 8, bd1 + ((kk * 2048) >> 4), I_MAT, 1);
          }
          tc::mma_commit(bar(c.a_done[buf]));
          if (pair) {
            tc::mma_commit(bar(c.empty[slot]));
            ++u;
            tc::mma_commit(bar(c.empty[slot2]));
            continue;
          }
        }
        tc::mma_commit(bar(c.empty[slot]));
      }
      // Drain: wait for every MMA issued so far before TMEM is released.
      tc::mma_commit(bar(c.drain));
      tc::wait_drain(bar(c.drain), 0, kWaitLimit);
    }
  }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 9) tc::tmem_dealloc(tmem, 512);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D map over a dense [d2][d1][d0] tensor of 16-bit elements, 128-byte swizzle,
// box {64, rows, 1}; reads past the end of d1 return zeros.
bool map3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
           uint64_t d2, uint32_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

template <int D, int BLK, int ORDER>
static cudaError_t launch_t(const ForwardArgs& a, cudaStream_t st) {
  Params p;
  const uint64_t bh = (uint64_t)a.B * a.H;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  bool ok = map3d(&p.tmQ, BF, a.q, D, a.Nq, bh, TQ) && map3d(&p.tmK, BF, a.k, D, a.Nk, bh, BLK) &&
            map3d(&p.tmV, HF, a.v, D, a.Nk, bh, BLK) &&
            map3d(&p.tmKb, BF, a.kbar16, D, a.nkb, 2 * bh, KC) &&
            map3d(&p.tmVs, HF, a.vsum16, D, a.nkb, bh, KC);
  if (ORDER == 1) ok = ok && map3d(&p.tmM, HF, a.M, D, D, bh * a.nkb, D);
  else p.tmM = p.tmVs;
  if (!ok) return cudaErrorInvalidValue;
  p.kv_idx = a.kv_idx;
  p.kv_cnt = a.kv_cnt;
  p.out = a.out;
  p.err_flag = a.err_flag;
  p.cap = a.cap;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.nqb = a.nqb;
  p.nkb = a.nkb;
  p.out_dtype = a.out_dtype;
  p.scale = a.scale;
  auto kern = forward_tc_kernel<D, BLK, ORDER>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((a.Nq + TQ - 1) / TQ, a.B * a.H);
  kern<<<grid, NTHREADS, SMEM_BYTES, st>>>(p);
  return cudaGetLastError();
}

}  // namespace tcf

cudaError_t launch_forward(const ForwardArgs& p, cudaStream_t st) {
#define SA_TC_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && p.order == O_) return tcf::launch_t<D_, B_, O_>(p, st);
  SA_TC_CASE(64, 64, 0) SA_TC_CASE(64, 64, 1) SA_TC_CASE(64, 128, 0) SA_TC_CASE(64, 128, 1)
  SA_TC_CASE(128, 64, 0) SA_TC_CASE(128, 64, 1) SA_TC_CASE(128, 128, 0) SA_TC_CASE(128, 128, 1)
#undef SA_TC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
