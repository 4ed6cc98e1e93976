// Forward pass on the 5th-generation tensor cores: tcgen05.mma with accumulators in
// tensor memory, operands staged by TMA, one warp-specialised CTA per two tiles of
// 128 query rows.
//
// Follows "PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion
// Transformers" §2: Algorithme Central (o_t = N_t / D_t; exact terms for the kept
// blocks; alpha_{t,j} (sum_n v_{j,n}) for the others; the first-order term, here per
// block: alpha_{t,j} * scale * q_t M_j) and Implémentation Matérielle (phase 1 exact
// tiles in on-chip memory, phase 2 a sweep over the aggregated block vectors, phase 3
// the first-order correction), all merged into one online softmax.
//
// Two query tiles per CTA. Neighbouring query blocks skip mostly the same key blocks,
// so every operand that TMA brings in (centroids, value sums, M_j, K, V) serves both
// tiles: half the L2 traffic per tensor-core flop of one tile per CTA. Each tile takes
// part only in the work items its own rows need.
//
// Roles (384 threads):
//   warps 0-3  softmax of tile 0, warps 4-7 softmax of tile 1: one thread per query
//              row (TMEM lane 32*(w%4) + lane). They read logits from TMEM, keep the
//              running max (rescaling O lazily, only when a row's max grows by more
//              than 2^11), write P back to TMEM as the A operand of the value product,
//              and build the order-1 operand A_j = (scale * alpha_tj) q_t in TMEM.
//   warp 8     TMA producer: both Q tiles once, then every operand through a ring of
//              4 x 32 KB units (each unit holds two 16 KB pieces or one M_j).
//   warps 9-10 one MMA-issuing thread per tile (warp 9 also allocates TMEM). Issuing
//              a 128x128x16 tcgen05.mma takes about as long as the tensor core takes to
//              run it, so one thread cannot also wait and commit without leaving the
//              pipe idle; two issuers keep it fed.
//   warp 11    idle (it completes the control warpgroup for the register split).
// TMEM columns: O_0 [0, 128), O_1 [128, 256); tile t owns two 64-column buffers at
// 256 + 128 t + 64 b (b = 0, 1). Every work item of a tile takes the tile's next
// buffer in turn: 64 logits (then their P as fp16), or one order-1 operand. The
// logits of a tile's next item are therefore computed while its softmax works on
// the current one, and one order-1 operand is built while the other is in use.
//
// Work items, in order (the same walk runs in every role):
//   TILE c   64 centroids (bf16 hi + lo) and value sums (fp16):
//            S_t = Q_t Kbar_hi^T + Q_t Kbar_lo^T, P_t, O_t += P_t Vsum
//   MAT j    each skipped block of the current centroid tile (order 1):
//            O_t += A_t,j M_j (fp16)
//   EXACT    each 64-key half (block 128) or block (block 64) of each kept block:
//            S_t = Q_t K^T (bf16), P_t, O_t += P_t V (fp16)
// For each tile, the logits of its next item are issued before the value product of
// its current one. Order-1 TILE items are an exception: their value product follows
// at once, because the order-1 operands of the centroid tile come next.
// Every mbarrier wait is bounded: on timeout the CTA sets err_flag, abandons its work,
// drains its own TMA loads and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace sa {
namespace tcf {

constexpr int TQ = 128;        // query rows per tile
constexpr int NT = 2;          // tiles per CTA
constexpr int KC = 64;         // centroids per TILE item; keys per EXACT item
constexpr int NU = 4;          // ring units
constexpr int UNIT = 32768;    // bytes per ring unit
constexpr int HALF = UNIT / 2; // bytes per piece slot
constexpr int MAXW = 64;       // bitmap words (2048 blocks)
constexpr int NSOFT = 256;     // softmax threads (2 warpgroups, one per tile)
constexpr int NTHREADS = NSOFT + 128;  // + one control warpgroup (producer, 2 MMA, 1 idle)
// Register split after launch (168 per thread at launch = 64,512 per CTA): the
// control warpgroup gives registers back, the softmax warpgroups take them.
constexpr int kRegCtl = 72, kRegSoft = 216;
static_assert(2 * 128 * kRegSoft + 128 * kRegCtl <= 168 * NTHREADS, "register split");
constexpr float kThresh = 11.0f;  // lazy-rescale threshold, base-2 units (P < 2^11)
constexpr float kF16Safe = 32768.f;  // bound kept on the fp16 order-1 operand (fp16 max 65504)
constexpr uint32_t kWaitLimit = 1u << 18;  // ~0.3 s: far above any legitimate wait

constexpr uint32_t COL_O = 0, COL_R = 256;

// shared-memory map (offsets from a 1024-aligned base)
constexpr int OFF_Q = 0;                        // Q tiles, bf16, swizzled (2 x 32 KB)
constexpr int OFF_U = 65536;                    // ring
constexpr int OFF_STASH = OFF_U + NU * UNIT;    // P of each tile's current centroid tile,
                                                // fp16 [tile][column][row] (32 KB)
constexpr int OFF_CTL = OFF_STASH + NT * 64 * TQ * 2;  // control block (2 KB)
constexpr int SMEM_BYTES = OFF_CTL + 2048 + 1024;

struct Params {
  CUtensorMap tmQ, tmK, tmV, tmKb, tmVs, tmM;
  const int32_t* kv_idx;
  const int32_t* kv_cnt;
  void* out;
  int32_t* err_flag;
  int cap, Nq, Nk, nqb, nkb, out_dtype;
  int nx, nbh;  // CTAs (pairs of query tiles) per (batch, head); batch x heads
  int nsplit;   // key-range splits per pair of query tiles (1: no split)
  float* part;  // nsplit > 1: partial results [nsplit][nbh][Nq][D] fp32, then (m, l) pairs
  float scale;
};

// The CTA's pair of query tiles, its (batch, head) and its key-range split. The grid is
// one-dimensional and puts every (batch, head)'s last pair, which may hold fewer rows,
// after all full pairs, so that the shorter CTAs fill the last wave. Neighbouring CTAs
// share (batch, head) and split, hence their keys and values in L2.
template <bool SPLIT>
SA_DEVI void cta_coords(const Params& p, int& x, int& bh, int& split) {
  const int L = blockIdx.x, nfull = p.nx - 1;
  if constexpr (!SPLIT) {
    split = 0;
    if (L < nfull * p.nbh) {
      x = L % nfull;
      bh = L / nfull;
    } else {
      x = p.nx - 1;
      bh = L - nfull * p.nbh;
    }
    return;
  }
  int r;
  if (L < nfull * p.nbh * p.nsplit) {
    x = L % nfull;
    r = L / nfull;
  } else {
    x = p.nx - 1;
    r = L - nfull * p.nbh * p.nsplit;
  }
  split = r % p.nsplit;
  bh = r / p.nsplit;
}

struct Ctl {  // control block in shared memory
  uint64_t full[NU], empty[NU];
  // per tile and TMEM buffer: logits landed, P written, order-1 operand written,
  // buffer released (the last product reading it is complete)
  uint64_t s_full[NT][2], p_full[NT][2], a_full[NT][2], rel[NT][2];
  uint64_t o_final[NT], q_full, init_done;
  int4 evq[NU];             // step record of the first ring unit of each step
  uint32_t tmem_base;
  int abort;
  int tvalid;               // bit t: tile t has rows below Nq
  uint32_t kept[NT][2][MAXW];  // kept blocks of each query block (half) of each tile
  int jlo, jhi, split;      // key blocks of this CTA's split: [jlo, jhi)
};
static_assert(sizeof(Ctl) <= 2048, "control block");

enum : int { kTile = 0, kMat = 1, kExact = 2, kNone = 3 };
struct Item {
  int kind, j;  // TILE: j = centroid-tile index; MAT / EXACT: j = block index
  int mask;     // bit t: tile t takes part
  int half;     // EXACT, block 128: which 64 keys of the block
};

// Key blocks [jlo, jhi) of a split: whole centroid tiles of KC blocks, shared out evenly.
SA_DEVI void split_range(int split, int nsplit, int nkb, int& jlo, int& jhi) {
  const int ntl = (nkb + KC - 1) / KC;
  jlo = min(nkb, (int)((long long)split * ntl / nsplit) * KC);
  jhi = min(nkb, (int)((long long)(split + 1) * ntl / nsplit) * KC);
}

// Blocks j of word w (j = 32 w + bit) inside the CTA's key range [jlo, jhi); without
// splits the range is [0, nkb) with jhi = nkb.
template <bool SPLIT>
SA_DEVI uint32_t range_bits(int w, int jlo, int jhi) {
  if constexpr (!SPLIT) {
    const int lo = w * 32;
    return lo + 32 <= jhi ? 0xffffffffu : (lo < jhi ? (1u << (jhi - lo)) - 1u : 0u);
  }
  const int a = max(jlo - 32 * w, 0), b = min(jhi - 32 * w, 32);
  if (b <= a) return 0u;
  return (b - a == 32 ? 0xffffffffu : (1u << (b - a)) - 1u) << a;
}
// Blocks of word w that some query block of tile t skips / keeps.
template <bool SPLIT>
SA_DEVI uint32_t skip_word(const Ctl& c, int t, int w, int jlo, int jhi) {
  if (!((c.tvalid >> t) & 1)) return 0u;
  return ~(c.kept[t][0][w] & c.kept[t][1][w]) & range_bits<SPLIT>(w, jlo, jhi);
}
template <bool SPLIT>
SA_DEVI uint32_t kept_word(const Ctl& c, int t, int w, int jlo, int jhi) {
  if (!((c.tvalid >> t) & 1)) return 0u;
  return (c.kept[t][0][w] | c.kept[t][1][w]) & range_bits<SPLIT>(w, jlo, jhi);
}
template <bool SPLIT>
SA_DEVI uint64_t skip64(const Ctl& c, int t, int ct, int jlo, int jhi) {
  return (uint64_t)skip_word<SPLIT>(c, t, 2 * ct, jlo, jhi) |
         ((uint64_t)skip_word<SPLIT>(c, t, 2 * ct + 1, jlo, jhi) << 32);
}

// The walk over work items; identical in every role. Union masks of the current
// centroid tile (phase 0) or 32-block word (phase 1) are held in registers. It covers
// the key blocks [jlo, jhi) of the CTA's split (every block when there is one split).
template <int BLK, bool SPLIT>
struct Walk {
  int phase = 0, tile = 0, word = -1, half = 0, jcur = 0, mcur = 0;
  int jlo = 0, jhi = 0;  // the split's key blocks, kept in registers
  SA_DEVI void start(const Ctl& c) {
    jlo = SPLIT ? c.jlo : 0;
    jhi = c.jhi;
    tile = jlo / KC;
    word = jlo / 32 - 1;
  }
  int gmask = 0;       // order 2: tiles with a skipped block so far
  bool in_tile = false, gdone = false;
  uint64_t tmask = 0, sk0 = 0, sk1 = 0;  // phase 0: union / per-tile skipped blocks
  uint32_t kmask = 0, kw0 = 0, kw1 = 0;  // phase 1: union / per-tile kept blocks
  template <int ORDER>
  SA_DEVI Item next(const Ctl& c, int nkb) {
    const int ntiles = (jhi + KC - 1) / KC;
    while (true) {
      if (phase == 0) {
        if (!in_tile) {
          if (tile >= ntiles) {
            if (ORDER == 2 && !gdone && gmask) {  // the global first-order item
              gdone = true;
              return Item{kMat, -1, gmask, 0};
            }
            phase = 1;
            continue;
          }
          sk0 = skip64<SPLIT>(c, 0, tile, jlo, jhi);
          sk1 = skip64<SPLIT>(c, 1, tile, jlo, jhi);
          tmask = sk0 | sk1;
          if (tmask) {
            in_tile = true;
            const int m = (sk0 != 0) | ((sk1 != 0) << 1);
            gmask |= m;
            return Item{kTile, tile, m, 0};
          }
          ++tile;
          continue;
        }
        if (ORDER == 1 && tmask) {  // skipped blocks of this centroid tile, one at a time
          const int c1 = __ffsll((long long)tmask) - 1;
          tmask &= tmask - 1;
          return Item{kMat, tile * KC + c1, (int)((sk0 >> c1) & 1u) | (int)(((sk1 >> c1) & 1u) << 1), 0};
        }
        in_tile = false;
        ++tile;
        continue;
      }
      if (BLK == 128 && half == 1) {  // second 64 keys of the current kept block
        half = 0;
        return Item{kExact, jcur, mcur, 1};
      }
      while (!kmask) {
        if (++word >= (jhi + 31) / 32) {
          word = (jhi + 31) / 32;  // stays at the end: later calls return kNone again
          return Item{kNone, 0, 0, 0};
        }
        kw0 = kept_word<SPLIT>(c, 0, word, jlo, jhi);
        kw1 = kept_word<SPLIT>(c, 1, word, jlo, jhi);
        kmask = kw0 | kw1;
      }
      const int b = __ffs(kmask) - 1;
      kmask &= kmask - 1;
      jcur = word * 32 + b;
      mcur = (int)((kw0 >> b) & 1u) | (int)(((kw1 >> b) & 1u) << 1);
      if (BLK == 128) half = 1;
      return Item{kExact, jcur, mcur, 0};
    }
  }
};

// Steps: what the producer loads into one or two ring units and the MMA threads then
// issue. A unit holds two 16 KB pieces (a 64-row K, V, centroid plane or value-sum
// tile) or one M_j. An SX step carries the logits of the next TILE/EXACT item and
// the value products of the previous one ("pending", one per tile that took part);
// its pieces are [V or Vsum of the pending item] + [K, or Kbar hi + lo, of the new].
enum : int { stSX = 0, stFlush = 1, stMat = 2, stEnd = 3 };
struct Step {
  int type, nunits;
  int cur_kind, cur_mask, cur_j, cur_half;      // SX: new TILE/EXACT item; MAT: the block
  int pend_kind, pend_mask, pend_j, pend_half;  // SX / FLUSH: item whose value products are due
};
template <int BLK, bool SPLIT>
struct StepGen {
  Walk<BLK, SPLIT> wk;
  int pend_kind = 0, pend_mask = 0, pend_j = 0, pend_half = 0;
  bool flush_next = false;
  template <int ORDER>
  SA_DEVI Step next(const Ctl& c, int nkb) {
    if (flush_next) {  // order 1: a TILE's value products come before its MAT items
      flush_next = false;
      const Step s{stFlush, 1, 0, 0, 0, 0, pend_kind, pend_mask, pend_j, pend_half};
      pend_mask = 0;
      return s;
    }
    const Item it = wk.template next<ORDER>(c, nkb);
    if (it.kind == kNone) {
      if (pend_mask) {
        const Step s{stFlush, 1, 0, 0, 0, 0, pend_kind, pend_mask, pend_j, pend_half};
        pend_mask = 0;
        return s;
      }
      return Step{stEnd, 1, 0, 0, 0, 0, 0, 0, 0, 0};
    }
    if (it.kind == kMat) return Step{stMat, 1, kMat, it.mask, it.j, 0, 0, 0, 0, 0};
    const int pieces = (pend_mask ? 1 : 0) + (it.kind == kTile ? 2 : 1);
    const Step s{stSX, (pieces + 1) / 2, it.kind, it.mask, it.j, it.half,
                 pend_kind, pend_mask, pend_j, pend_half};
    pend_kind = it.kind;
    pend_mask = it.mask;
    pend_j = it.j;
    pend_half = it.half;
    if (ORDER >= 1 && it.kind == kTile) flush_next = true;
    return s;
  }
};
SA_DEVI int encode(const Step& s) {
  return s.type | (s.cur_kind << 4) | (s.pend_kind << 8) | (s.cur_mask << 12) | (s.pend_mask << 14) |
         (s.nunits << 16);
}

template <int D, int BLK>
struct Bytes {
  static constexpr int SUB = D / 64;                    // 64-column sub-tiles per row
  static constexpr uint32_t PIECE = SUB * 64 * 128;     // 64 rows: K, V, Kbar plane, Vsum
  static constexpr uint32_t M = SUB * D * 128;          // one M_j
  static constexpr uint32_t Q = SUB * TQ * 128;         // one query tile
  static_assert(PIECE <= HALF && M <= UNIT, "ring pieces");
};

// Softmax warpgroup of tile t = warp / 4. Thread (warp w, lane l) owns query row
// r = 32*(w%4) + l of the tile: all its logits, its running max and sum, its O row.
template <int D, int BLK, int ORDER, bool SPLIT>
SA_DEVI void softmax_role(const Params& p, Ctl& c, uint8_t* gbase, uint32_t tmem, tc::Waiter& wt,
                          int warp, int lane, int cx, int bh) {
  using By = Bytes<D, BLK>;
  constexpr int QW = D / 2;  // fp16 pairs per query row
  const int t = warp >> 2, qw = warp & 3;
  const int r = 32 * qw + lane;
  const uint32_t lane_off = (uint32_t)(32 * qw) << 16;
  const uint32_t rt = tmem + lane_off + COL_R + 128 * t;  // buffer 0 of this tile
  const uint32_t ot = tmem + lane_off + COL_O + 128 * t;  // O rows
  const int h = BLK == 64 ? (r >> 6) : 0;                  // query block of the row
  const float sl2 = p.scale * kLog2e;
  const int nkb = p.nkb;
  const int row0 = cx * (NT * TQ) + t * TQ;
  const uint32_t* kept_h = c.kept[t][h];
  const int jlo = c.jlo, jhi = c.jhi;  // the CTA's key blocks (split)
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };
  auto uni = [](bool x) { return __all_sync(0xffffffffu, x); };
  // One arrival per warp: every lane's tensor-memory stores are ordered before the
  // warp barrier, and lane 0 arrives after it.
  auto warp_arrive = [&](uint32_t b) {
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(b);
  };

  bool ok = uni(wt.wait(bar(c.q_full), 0, 9));
  // fp16 copy of this thread's Q row, in registers (order-1 operands)
  uint32_t q16[ORDER >= 1 ? QW : 1];
  float qmax = 0.f;  // largest |q| of the row (keeps the order-1/2 operands in fp16 range)
  if constexpr (ORDER >= 1) {
#pragma unroll
    for (int i = 0; i < QW / 4; ++i) {
      const int s = i / 8, cw = i % 8;
      const uint32_t off = t * By::Q + s * TQ * 128 + r * 128 + ((cw ^ (r & 7)) << 4);
      const uint4 x = *reinterpret_cast<const uint4*>(gbase + OFF_Q + off);
      q16[4 * i + 0] = bf16x2_to_f16x2(x.x);
      q16[4 * i + 1] = bf16x2_to_f16x2(x.y);
      q16[4 * i + 2] = bf16x2_to_f16x2(x.z);
      q16[4 * i + 3] = bf16x2_to_f16x2(x.w);
    }
  }
  {
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) tc::tmem_st32(ot + 32 * k, z);
    tc::tmem_wait_st();
  }
  if constexpr (ORDER >= 1) {
#pragma unroll
    for (int i = 0; i < QW; ++i) {
      const __half2 h = *reinterpret_cast<const __half2*>(&q16[i]);
      qmax = fmaxf(qmax, fmaxf(fabsf(__low2float(h)), fabsf(__high2float(h))));
    }
  }
  warp_arrive(bar(c.init_done));
  // Order 1 builds (scale * alpha) q_t in fp16 with alpha < 2^thr (the rescale threshold):
  // a row with large |q| lowers its threshold so that the operand stays below 2^15. For
  // |q| up to 2^15 / (2^11 scale) (181 at d = 128) the threshold stays 2^11.
  float thr = kThresh;
  if constexpr (ORDER == 1) {
    if (p.scale * qmax * exp2f(kThresh) > kF16Safe) {
      int e;  // kF16Safe / (scale qmax) = m 2^e with m in [0.5, 1): floor(log2) = e - 1
      frexpf(kF16Safe / (p.scale * qmax), &e);
      thr = fmaxf(0.f, (float)(e - 1));
    }
  }

  float m_ref = -INFINITY, l = 0.f;
  float asum = 0.f;          // order 2: sum of the skipped blocks' alpha, relative to m_ref
  int n = 0;                 // items of this tile so far; item n uses buffer n & 1
  // Per-buffer phase parities as bit masks (bit b for buffer b): next s_full wait;
  // number of items so far (rel phases); whether the buffer has been used.
  uint32_t sph = 0, rcnt = 0, rany = 0;
  // P of the current centroid tile, this thread's row: stash[c * TQ] is column c
  uint16_t* stash = reinterpret_cast<uint16_t*>(gbase + OFF_STASH) + t * 64 * TQ + r;
  const uint64_t sl2x2 = tc::f2(sl2, sl2);

  // One TILE or EXACT item: this thread's 64 logits in buffer b.
  auto s_item = [&](const Item& it, auto tile_tag) __attribute__((always_inline)) -> bool {
    constexpr bool TILE = decltype(tile_tag)::value;
    const int idx = n++;
    const int b = idx & 1;
    const uint32_t buf = rt + 64 * b;
    if (!uni(wt.fast(bar(c.s_full[t][b]), (sph >> b) & 1, 11))) return false;
    sph ^= 1u << b;
    rcnt ^= 1u << b;
    rany |= 1u << b;
    tc::fence_after_sync();
    uint32_t mbits[2];
    bool masked = TILE;  // the same for the whole warp
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (TILE) {
        // a centroid column counts for the rows whose query block skips its block
        const int w = (it.j * KC + 32 * k) >> 5;
        mbits[k] = ~kept_h[w] & range_bits<SPLIT>(w, jlo, jhi);
      } else {
        const int t0 = it.j * BLK + 64 * it.half + 32 * k;
        mbits[k] = t0 + 32 <= p.Nk ? 0xffffffffu : (t0 < p.Nk ? (1u << (p.Nk - t0)) - 1u : 0u);
        if (BLK == 64 && !((kept_h[it.j >> 5] >> (it.j & 31)) & 1u)) mbits[k] = 0u;
        masked = masked || mbits[k] != 0xffffffffu;
      }
    }
    // Raw logits; masked columns become -inf, which the exponential maps to an exact
    // zero. A TILE's logits are read twice from TMEM (max, then exponentials), 32 at
    // a time, which keeps registers free for the order-1 state; an EXACT item's 64 are
    // read once.
    constexpr int NR = TILE ? 32 : 64;
    float xv[NR];
    auto fetch = [&, masked](int k0) __attribute__((always_inline)) {
      uint32_t sv[NR];
#pragma unroll
      for (int k = 0; k < NR / 32; ++k) tc::tmem_ld32(buf + 32 * (k0 + k), sv + 32 * k);
      tc::tmem_wait_ld();
      if (masked) {
#pragma unroll
        for (int k = 0; k < NR / 32; ++k)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            xv[32 * k + i] = ((mbits[k0 + k] >> i) & 1u) ? __uint_as_float(sv[32 * k + i]) : -INFINITY;
      } else {
#pragma unroll
        for (int i = 0; i < NR; ++i) xv[i] = __uint_as_float(sv[i]);
      }
    };
    // row max of the raw logits (the scale is positive), in base-2 units after scaling
    float mx = -INFINITY;
#pragma unroll
    for (int k0 = 0; k0 < 2; k0 += NR / 32) {
      fetch(k0);
      float m8[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) m8[a] = tc::max3(xv[a], xv[8 + a], xv[16 + a]);
#pragma unroll
      for (int a = 0; a < 8; ++a) m8[a] = NR == 64 ? tc::max3(m8[a], xv[24 + a], xv[(32 + a) % NR]) : fmaxf(m8[a], xv[24 + a]);
      if (NR == 64) {
#pragma unroll
        for (int a = 0; a < 8; ++a) m8[a] = tc::max3(m8[a], xv[(40 + a) % NR], xv[(48 + a) % NR]);
#pragma unroll
        for (int a = 0; a < 8; ++a) m8[a] = fmaxf(m8[a], xv[(56 + a) % NR]);
      }
      mx = tc::max3(mx, tc::max3(tc::max3(m8[0], m8[1], m8[2]), tc::max3(m8[3], m8[4], m8[5]), m8[6]), m8[7]);
    }
    mx *= sl2;
    // Lazy rescale: only rows whose max grew by more than 2^thr move their
    // reference; rows that had no reference yet just take one (O is still zero).
    const bool grow = mx > m_ref + thr;
    const bool need_o = grow && m_ref != -INFINITY;
    const float f = need_o ? tc::ex2(m_ref - mx) : 1.f;
    if (grow) m_ref = mx;
    // A row with no unmasked logit so far keeps m_ref = -inf; its P must be 0, not NaN.
    const float mr = m_ref == -INFINITY ? 0.f : m_ref;
    const uint64_t nmr2 = tc::f2(-mr, -mr);
    // P = 2^(x * scale * log2(e) - m_ref) as fp16 pairs, written over the logits
    // already read; row sums in two packed accumulators.
    uint64_t acc0 = tc::f2(0.f, 0.f), acc1 = acc0;
    // TILE: column of the possibly partial last block, and its P
    const int jl = TILE ? nkb - 1 - it.j * KC : -1;
    float plast = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (TILE) fetch(k);
      const float* xk = TILE ? xv : xv + 32 * k;
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const uint64_t y = tc::fma2(tc::f2(xk[i], xk[i + 1]), sl2x2, nmr2);
        float y0, y1;
        tc::f2_split(y, y0, y1);
        const float x0 = tc::ex2(y0), x1 = tc::ex2(y1);
        const uint64_t ev = tc::f2(x0, x1);
        if ((i / 2) & 1) acc1 = tc::add2(acc1, ev); else acc0 = tc::add2(acc0, ev);
        pk[i / 2] = pack_f16(x0, x1);
        if (TILE) plast = (32 * k + i == jl) ? x0 : ((32 * k + i + 1 == jl) ? x1 : plast);
      }
      if constexpr (TILE && ORDER == 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          stash[(32 * k + 2 * i) * TQ] = (uint16_t)(pk[i] & 0xffffu);
          stash[(32 * k + 2 * i + 1) * TQ] = (uint16_t)(pk[i] >> 16);
        }
      }
      tc::tmem_st16(buf + 16 * k, pk);
    }
    // O_t rescale, once the products into O_t issued so far are complete: the last
    // one is the previous item's (value product or order-1 product), released on the
    // other buffer; the value product of this item waits for p_full.
    bool waited = true;
    if (__any_sync(0xffffffffu, need_o)) {
      if (idx > 0) {
        waited = uni(wt.fast(bar(c.rel[t][1 - b]), ((rcnt >> (1 - b)) & 1) ^ 1, 12));
        tc::fence_after_sync();
      }
#pragma unroll
      for (int k = 0; k < D / 32 && waited; ++k) {
        uint32_t v[32];
        tc::tmem_ld32(ot + 32 * k, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
        tc::tmem_st32(ot + 32 * k, v);
      }
    }
    float a0, a1, a2, a3;
    tc::f2_split(acc0, a0, a1);
    tc::f2_split(acc1, a2, a3);
    float ls = (a0 + a1) + (a2 + a3);
    if (ORDER == 2 && TILE) asum = asum * f + ls;  // alpha of the skipped blocks (P is 0 elsewhere)
    // order-0 denominator weight n_j: b for every block but a partial last one
    if (TILE) ls = ls * (float)BLK + plast * (float)(p.Nk - nkb * BLK);
    l = l * f + ls;
    tc::tmem_wait_st();
    if (!waited) return false;
    warp_arrive(bar(c.p_full[t][b]));
    return true;
  };

  Walk<BLK, SPLIT> wk;
  wk.start(c);
  Item it{kNone, 0, 0, 0};
  int cur_tile = 0;
  // ---- phase 0: centroid tiles and their order-1 products ----
  while (ok) {
    it = wk.template next<ORDER>(c, nkb);
    if (it.kind == kExact || it.kind == kNone) break;
    if (!((it.mask >> t) & 1)) continue;
    if (it.kind == kTile) {
      ok = s_item(it, std::true_type{});
      cur_tile = it.j;
      continue;
    }
    if constexpr (ORDER >= 1) {
      // The operand does not depend on the buffer: compute (its first 32 columns)
      // first, then wait until the products that last read the buffer (two items
      // back) are complete.
      float as;  // scale * alpha of the item's row
      if constexpr (ORDER == 1) {
        as = __half2float(__ushort_as_half(stash[(it.j - cur_tile * KC) * TQ])) * p.scale;
      } else {
        // The global item: A = (scale * sum_j alpha_tj) q_t must stay in fp16 range. A row
        // whose operand would exceed 2^14 moves its reference up by E (a rescale by 2^-E
        // of O, l and the alpha sum, as when its max grows), after the last product into
        // O_t (the previous item's) is complete.
        const float g = asum * p.scale * qmax;
        const int E = g > 16384.f ? (int)ceilf(log2f(g * (1.f / 16384.f))) : 0;
        if (__any_sync(0xffffffffu, E > 0)) {
          const float f = exp2f((float)-E);
          if (n > 0) {
            const int pb = (n - 1) & 1;
            ok = uni(wt.fast(bar(c.rel[t][pb]), ((rcnt >> pb) & 1) ^ 1, 12));
            tc::fence_after_sync();
          }
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < D / 32; ++k) {
            uint32_t v[32];
            tc::tmem_ld32(ot + 32 * k, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
            tc::tmem_st32(ot + 32 * k, v);
          }
          tc::tmem_wait_st();
          m_ref += (float)E;
          l *= f;
          asum *= f;
        }
        as = asum * p.scale;
      }
      const __half2 al = __float2half2_rn(as);
      auto part = [&](int k, uint32_t* a) __attribute__((always_inline)) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const __half2 y = __hmul2(*reinterpret_cast<const __half2*>(&q16[32 * k + i]), al);
          a[i] = *reinterpret_cast<const uint32_t*>(&y);
        }
      };
      uint32_t a[32];
      part(0, a);
      const int b = n & 1;
      ++n;
      if ((rany >> b) & 1) ok = uni(wt.fast(bar(c.rel[t][b]), ((rcnt >> b) & 1) ^ 1, 10));
      rcnt ^= 1u << b;
      rany |= 1u << b;
      if (!ok) break;
      tc::fence_after_sync();
      tc::tmem_st32(rt + 64 * b, a);
#pragma unroll
      for (int k = 1; k < QW / 32; ++k) {
        part(k, a);
        tc::tmem_st32(rt + 64 * b + 32 * k, a);
      }
      tc::tmem_wait_st();
      warp_arrive(bar(c.a_full[t][b]));
    }
  }
  // ---- phase 1: kept blocks ----
  while (ok && it.kind == kExact) {
    if ((it.mask >> t) & 1) ok = s_item(it, std::false_type{});
    it = wk.template next<ORDER>(c, nkb);
  }

  // ---- epilogue: O / l ----
  if (ok) ok = uni(wt.wait(bar(c.o_final[t]), 0, 13));
  tc::fence_after_sync();
  if (!ok) return;
  const bool store = row0 + r < p.Nq;
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const size_t rowoff = ((size_t)bh * p.Nq + row0 + (store ? r : 0)) * D;
  if constexpr (SPLIT) {
    // A split's partial result: O relative to 2^m_ref, not yet divided, with (m_ref, l).
    const size_t prow = ((size_t)c.split * p.nbh + bh) * p.Nq + row0 + (store ? r : 0);
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      uint32_t v[32];
      tc::tmem_ld32(ot + 32 * k, v);
      tc::tmem_wait_ld();
      if (!store) continue;
      float4* o = reinterpret_cast<float4*>(p.part + prow * D + 32 * k);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                           __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    }
    if (store)
      reinterpret_cast<float2*>(p.part + (size_t)p.nsplit * p.nbh * p.Nq * D)[prow] =
          make_float2(m_ref, l);
  } else {
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      uint32_t v[32];
      tc::tmem_ld32(ot + 32 * k, v);
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
}

template <int D, int BLK, int ORDER, bool SPLIT>
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
  int cx, bh, split;
  cta_coords<SPLIT>(p, cx, bh, split);
  const int q0 = cx * (NT * TQ);
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
      tc::mbar_init(bar(c.empty[u]), NT);  // one release per MMA thread
    }
    for (int t = 0; t < NT; ++t) {
      tc::mbar_init(bar(c.o_final[t]), 1);
      for (int b = 0; b < 2; ++b) {
        tc::mbar_init(bar(c.s_full[t][b]), 1);
        tc::mbar_init(bar(c.rel[t][b]), 1);
        tc::mbar_init(bar(c.p_full[t][b]), 4);
        tc::mbar_init(bar(c.a_full[t][b]), 4);
      }
    }
    tc::mbar_init(bar(c.q_full), 1);
    tc::mbar_init(bar(c.init_done), NSOFT / 32);
    tc::fence_mbar_init();
    tc::fence_proxy_async();
  }
  if (warp == 9) {
    tc::tmem_alloc(smem_u32(&c.tmem_base), 512);
    tc::tmem_relinquish();
  }
  if (warp < 8) {
    // Kept bitmaps of the query blocks of both tiles: one per tile (block 128) or
    // two (block 64, one per 64-row half).
    for (int w = tid; w < NT * 2 * MAXW; w += NSOFT) (&c.kept[0][0][0])[w] = 0u;
    asm volatile("bar.sync 1, %0;\n" ::"n"(NSOFT) : "memory");
    for (int t = 0; t < NT; ++t)
      for (int hh = 0; hh < (BLK == 64 ? 2 : 1); ++hh) {
        const int r0 = q0 + t * TQ + hh * 64;
        if (r0 >= p.Nq) continue;
        const size_t row = (size_t)bh * p.nqb + r0 / BLK;
        const int n = min(max(p.kv_cnt[row], 0), p.cap);
        const int32_t* src = p.kv_idx + row * p.cap;
        for (int x = tid; x < n; x += NSOFT) {
          const int j = src[x];
          if (j >= 0 && j < nkb) atomicOr(&c.kept[t][hh][j >> 5], 1u << (j & 31));
        }
      }
    asm volatile("bar.sync 1, %0;\n" ::"n"(NSOFT) : "memory");
    // a half without a query block of its own (block 128, or past Nq) repeats half 0
    for (int w = tid; w < NT * MAXW; w += NSOFT) {
      const int t = w / MAXW, ww = w % MAXW;
      if (BLK == 128 || q0 + t * TQ + 64 >= p.Nq) c.kept[t][1][ww] = c.kept[t][0][ww];
    }
    if (tid == 0) {
      c.tvalid = (q0 < p.Nq ? 1 : 0) | (q0 + TQ < p.Nq ? 2 : 0);
      split_range(split, p.nsplit, nkb, c.jlo, c.jhi);
      c.split = split;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = c.tmem_base;
  tc::Waiter wt{&c.abort, p.err_flag, kWaitLimit};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegSoft));
    softmax_role<D, BLK, ORDER, SPLIT>(p, c, gbase, tmem, wt, warp, lane, cx, bh);
  } else {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegCtl));
  if (warp == 8) {
    // =========================== TMA producer ===========================
    if (lane == 0) {
      tc::prefetch_tmap(&p.tmQ);
      const int ntq = q0 + TQ < p.Nq ? 2 : 1;
      tc::mbar_arrive_expect_tx(bar(c.q_full), ntq * By::Q);
      for (int t = 0; t < ntq; ++t)
        for (int s = 0; s < SUB; ++s)
          tc::tma_load_3d(base + OFF_Q + t * By::Q + s * TQ * 128, &p.tmQ, bar(c.q_full), 64 * s,
                          q0 + t * TQ, bh);
      StepGen<BLK, SPLIT> gen;
      gen.wk.start(c);
      int u = 0;
      bool ok = true;
      while (ok) {
        const Step s = gen.template next<ORDER>(c, nkb);
        for (int i = 0; i < s.nunits && ok; ++i) {
          const int v = u + i;
          if (v >= NU) ok = wt.fast(bar(c.empty[v % NU]), ((v / NU) - 1) & 1, 1);
        }
        if (!ok) break;
        const int slot = u % NU;
        const uint32_t fb = bar(c.full[slot]);
        // The MMA threads read the record after the unit's full barrier.
        c.evq[slot] = make_int4(encode(s), s.cur_j, s.pend_j, 0);
        if (s.type == stEnd) {
          tc::mbar_arrive(fb);  // terminal record, no data
          ++u;
          break;
        }
        // piece slot k of the step: unit k / 2, half k % 2
        auto piece = [&](int k) { return base + OFF_U + ((u + k / 2) % NU) * UNIT + (k % 2) * HALF; };
        uint32_t bytes = 0;
        if (s.type == stMat) bytes = By::M;
        else bytes = By::PIECE * ((s.pend_mask ? 1 : 0) + (s.type == stSX ? (s.cur_kind == kTile ? 2 : 1) : 0));
        // every load of the step completes on the first unit's barrier
        tc::mbar_arrive_expect_tx(fb, bytes);
        int k = 0;
        if (s.type == stMat) {
          // order 1: M_j of the head; order 2: the head's global matrix
          const int mz = ORDER == 2 ? bh : bh * nkb + s.cur_j;
          for (int x = 0; x < SUB; ++x)
            tc::tma_load_3d(piece(0) + x * D * 128, &p.tmM, fb, 64 * x, 0, mz);
        } else {
          if (s.pend_mask) {  // values of the pending item
            if (s.pend_kind == kTile) {
              for (int x = 0; x < SUB; ++x)
                tc::tma_load_3d(piece(0) + x * 64 * 128, &p.tmVs, fb, 64 * x, s.pend_j * KC, bh);
            } else {
              for (int x = 0; x < SUB; ++x)
                tc::tma_load_3d(piece(0) + x * 64 * 128, &p.tmV, fb, 64 * x,
                                s.pend_j * BLK + 64 * s.pend_half, bh);
            }
            k = 1;
          }
          if (s.type == stSX) {  // keys of the new item
            if (s.cur_kind == kTile) {
              for (int pl = 0; pl < 2; ++pl)
                for (int x = 0; x < SUB; ++x)
                  tc::tma_load_3d(piece(k + pl) + x * 64 * 128, &p.tmKb, fb, 64 * x, s.cur_j * KC,
                                  2 * bh + pl);
            } else {
              for (int x = 0; x < SUB; ++x)
                tc::tma_load_3d(piece(k) + x * 64 * 128, &p.tmK, fb, 64 * x,
                                s.cur_j * BLK + 64 * s.cur_half, bh);
            }
          }
        }
        // the second unit's barrier only keeps its phase count in step
        if (s.nunits == 2) tc::mbar_arrive(bar(c.full[(u + 1) % NU]));
        u += s.nunits;
      }
      // Drain: every load issued must land before the CTA exits.
      tc::wait_drain(bar(c.q_full), 0, kWaitLimit);
      for (int v = max(0, u - NU); v < u; ++v)
        tc::wait_drain(bar(c.full[v % NU]), (v / NU) & 1, kWaitLimit);
    }
  } else if (warp == 9 || warp == 10) {
    // ===================== MMA issuers: warp 9 + t for tile t =====================
    if (lane == 0) {
      const int t = warp - 9;
      constexpr uint32_t I_S = tc::idesc_f16(1, 1, 0, 64);
      constexpr uint32_t I_PV = tc::idesc_f16(0, 0, 1, D);
      bool ok = wt.wait(bar(c.init_done), 0, 2) && wt.wait(bar(c.q_full), 0, 3);
      tc::fence_after_sync();
      const uint32_t o_t = tmem + COL_O + 128 * t, r_t = tmem + COL_R + 128 * t;
      // Descriptor base of Q_t; per k-step only the start-address field (low bits) moves.
      const uint64_t dq = tc::sdesc(base + OFF_Q + t * By::Q, 16, 1024);
      int n = 0;                // items of this tile; item n uses buffer n & 1
      uint32_t pph = 0, aph = 0;  // p_full / a_full phase parities, bit b for buffer b
      int pbuf = 0;             // buffer of this tile's pending item
      for (int u = 0; ok;) {
        const int slot = u % NU;
        ok = wt.fast(bar(c.full[slot]), (u / NU) & 1, 4);
        if (!ok) break;
        const int rec = c.evq[slot].x;  // ordered by the full-barrier wait (asm with memory clobber)
        const int type = rec & 15, ck = (rec >> 4) & 15;
        const int cm = (rec >> 12) & 3, pm = (rec >> 14) & 3, nun = (rec >> 16) & 3;
        if (type == stEnd) break;
        const int slot2 = (u + 1) % NU;
        auto piece = [&](int k) {
          return base + OFF_U + (k / 2 ? slot2 : slot) * UNIT + (k % 2) * HALF;
        };
        bool issued = false;
        if (type == stMat) {
          if ((cm >> t) & 1) {
            const int b = n & 1;
            ++n;
            ok = wt.fast(bar(c.a_full[t][b]), (aph >> b) & 1, 7);
            aph ^= 1u << b;
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t b0 = tc::sdesc(piece(0), D * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              tc::mma_ts(o_t, r_t + 64 * b + kk * 8, b0 + ((kk * 2048) >> 4), I_PV, 1);
            tc::mma_commit(bar(c.rel[t][b]));
            issued = true;
          }
        } else {
          const int kp = pm ? 1 : 0;  // piece of the new item's keys
          int nbuf = pbuf;
          // logits of the new item first, into this tile's next buffer
          if (type == stSX && ((cm >> t) & 1)) {
            const int b = n & 1;
            ++n;
            const uint32_t dt = r_t + 64 * b;
            const int planes = ck == kTile ? 2 : 1;  // centroids: hi plane, then lo plane
            for (int pl = 0; pl < planes; ++pl) {
              const uint64_t bd = tc::sdesc(piece(kp + pl), 16, 1024);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t aoff = ((kk / 4) * TQ * 128 + (kk % 4) * 32) >> 4;
                const uint32_t boff = ((kk / 4) * 64 * 128 + (kk % 4) * 32) >> 4;
                tc::mma_ss(dt, dq + aoff, bd + boff, I_S, (pl | kk) > 0);
              }
            }
            tc::mma_commit(bar(c.s_full[t][b]));
            nbuf = b;
            issued = true;
          }
          // then the value product of the pending item, once its P is written
          if ((pm >> t) & 1) {
            ok = wt.fast(bar(c.p_full[t][pbuf]), (pph >> pbuf) & 1, 6);
            pph ^= 1u << pbuf;
            if (!ok) break;
            tc::fence_after_sync();
            const uint64_t bd = tc::sdesc(piece(0), 64 * 128, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc::mma_ts(o_t, r_t + 64 * pbuf + kk * 8, bd + ((kk * 2048) >> 4), I_PV, 1);
            tc::mma_commit(bar(c.rel[t][pbuf]));
            issued = true;
          }
          pbuf = nbuf;
        }
        // Release the step's units: after this thread's products have read them, or at
        // once if it issued none.
        if (issued) {
          tc::mma_commit(bar(c.empty[slot]));
          if (nun == 2) tc::mma_commit(bar(c.empty[slot2]));
        } else {
          tc::mbar_arrive(bar(c.empty[slot]));
          if (nun == 2) tc::mbar_arrive(bar(c.empty[slot2]));
        }
        u += nun;
      }
      // Every MMA this thread issued is complete once o_final[t] fires: the softmax
      // warps of tile t read O_t after it, and TMEM is released after it.
      tc::mma_commit(bar(c.o_final[t]));
      tc::wait_drain(bar(c.o_final[t]), 0, kWaitLimit);
    }
  }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 9) tc::tmem_dealloc(tmem, 512);
}


// Merge of the key-range splits of every query row: with M = max_s m_s and
// w_s = 2^(m_s - M), O = sum_s w_s O_s / sum_s w_s l_s (0 for a row with no weight).
// One warp per row; lane l holds D / 32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ part, int nsplit,
                                                      long long rows, void* out, int out_dtype) {
  constexpr int V = D / 32;
  static_assert(V == 2 || V == 4, "combine: d = 64 or 128");
  const long long row = (long long)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const float2* ml = reinterpret_cast<const float2*>(part + (size_t)nsplit * rows * D);
  float M = -INFINITY;
  for (int sp = 0; sp < nsplit; ++sp) M = fmaxf(M, ml[(size_t)sp * rows + row].x);
  float acc[V], L = 0.f;
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (M != -INFINITY) {
    for (int sp = 0; sp < nsplit; ++sp) {
      const float2 x = ml[(size_t)sp * rows + row];
      if (x.x == -INFINITY) continue;
      const float w = exp2f(x.x - M);
      L += w * x.y;
      // a lane's V consecutive columns in one 16- (V = 4) or 8-byte load: rows of D floats
      // in a 16-byte aligned buffer
      const float* o = part + ((size_t)sp * rows + row) * D + V * lane;
      if constexpr (V == 4) {
        const float4 y = *reinterpret_cast<const float4*>(o);
        acc[0] += w * y.x; acc[1] += w * y.y; acc[2] += w * y.z; acc[3] += w * y.w;
      } else {
        const float2 y = *reinterpret_cast<const float2*>(o);
        acc[0] += w * y.x; acc[1] += w * y.y;
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (out_dtype == 0) {
    float* o = static_cast<float*>(out) + (size_t)row * D + V * lane;
    if constexpr (V == 4) *reinterpret_cast<float4*>(o) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    else *reinterpret_cast<float2*>(o) = make_float2(acc[0] * inv, acc[1] * inv);
  } else {
    uint16_t* o = static_cast<uint16_t*>(out) + (size_t)row * D + V * lane;
    if constexpr (V == 4) *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
    else *reinterpret_cast<uint32_t*>(o) = pack_bf16(acc[0] * inv, acc[1] * inv);
  }
}

template <int D, int BLK, int ORDER>
static cudaError_t launch_t(const ForwardArgs& a, cudaStream_t st) {
  Params p;
  const uint64_t bh = (uint64_t)a.B * a.H;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  bool ok = map3d(&p.tmQ, BF, a.q, D, a.Nq, bh, TQ) && map3d(&p.tmK, BF, a.k, D, a.Nk, bh, 64) &&
            map3d(&p.tmV, HF, a.v, D, a.Nk, bh, 64) &&
            map3d(&p.tmKb, BF, a.kbar16, D, a.nkb, 2 * bh, KC) &&
            map3d(&p.tmVs, HF, a.vsum16, D, a.nkb, bh, KC);
  if (ORDER == 1) ok = ok && map3d(&p.tmM, HF, a.M, D, D, bh * a.nkb, D);
  else if (ORDER == 2) ok = ok && map3d(&p.tmM, HF, a.M, D, D, bh, D);
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
  p.nx = (a.Nq + NT * TQ - 1) / (NT * TQ);
  p.nbh = (int)bh;
  p.nsplit = a.splits > 1 ? a.splits : 1;
  p.part = p.nsplit > 1 ? a.work : nullptr;
  if (p.nsplit > 1 && !p.part) return cudaErrorInvalidValue;
  if ((uint64_t)p.nx * bh * p.nsplit > 0x7fffffffull) return cudaErrorInvalidValue;
  auto kern = p.nsplit > 1 ? forward_tc_kernel<D, BLK, ORDER, true>
                            : forward_tc_kernel<D, BLK, ORDER, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nx * p.nbh * p.nsplit);
  kern<<<grid, NTHREADS, SMEM_BYTES, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.nsplit == 1) return e;
  const long long rows = (long long)bh * a.Nq;
  combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p.part, p.nsplit, rows, a.out,
                                                                a.out_dtype);
  return cudaGetLastError();
}

}  // namespace tcf

cudaError_t launch_forward(const ForwardArgs& p, cudaStream_t st) {
#define SA_TC_CASE(D_, B_, O_) \
  if (p.d == D_ && p.block == B_ && p.order == O_) return tcf::launch_t<D_, B_, O_>(p, st);
  SA_TC_CASE(64, 64, 0) SA_TC_CASE(64, 64, 1) SA_TC_CASE(64, 64, 2)
  SA_TC_CASE(64, 128, 0) SA_TC_CASE(64, 128, 1) SA_TC_CASE(64, 128, 2)
  SA_TC_CASE(128, 64, 0) SA_TC_CASE(128, 64, 1) SA_TC_CASE(128, 64, 2)
  SA_TC_CASE(128, 128, 0) SA_TC_CASE(128, 128, 1) SA_TC_CASE(128, 128, 2)
#undef SA_TC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sa
