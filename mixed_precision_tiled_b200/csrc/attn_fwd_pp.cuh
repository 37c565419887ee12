// Routed mixed-precision attention forward, head dimension 128, INT8 8-bit format: two query
// tiles in flight per CTA, one softmax warpgroup each.  (FP8 E4M3 runs in the single-tile
// kernel of attn_fwd.cuh.)
//
// Same computation as attn_fwd.cuh (TileMix page, section 2 "How It Works": 8-bit or 16-bit
// score tiles chosen per tile, one shared online softmax; LampAttention abstract: 8-bit
// products, look-ahead recomputation of sensitive tiles in 16 bits), organised for B200 so
// that the tensor core works on one query tile while the softmax works on the other:
//   * persistent CTAs (one per SM) walk the work items longest first, in a fixed snake
//     order, or (when the KV planes exceed L2) take them from a launch-wide ticket counter in
//     an order that keeps the K/V planes in flight within L2;
//     an item is two 128-row query tiles X = 0, 1 that read the same K/V: the same query tile
//     of two heads of one KV group (grouped-query attention with an even group), otherwise two
//     query tiles of one head.  Each key tile is streamed through shared memory once for both:
//     K8 tiles in a ring of 16 KB slots, K16 and V tiles in a ring of 32 KB slots;
//   * TMEM holds S_0, S_1 (128 columns each) and O_0, O_1 (128 each) = all 512 columns;
//   * warpgroup X runs the softmax of query tile X (one row per thread, the row is the TMEM
//     lane); warp 8 issues TMA loads, warp 9 issues the MMAs (warp-wide loop, one elected
//     lane) in the order
//       S_0(0) S_1(0) | PV_0(t) S_0(t+1) PV_1(t) S_1(t+1) | ...
//     so that while one warpgroup exponentiates tile t, the tensor core runs the other tile's
//     P.V and next QK^T; P.V is issued in two halves as the softmax publishes them, and the
//     next item's Q loads and first QK^T overlap the current item's last tiles and epilogue;
//   * softmax arithmetic: exact int32 -> fp32 conversion (exact below 2^24), packed f32x2
//     FMAs / adds, 3-input max, the rounded row sum by mixed-precision adds of the packed
//     16-bit P, and a lazy O rescale: the reference max used for the exponentials only moves
//     when a row max exceeds it by more than 8 (log2 units), which keeps P <= 256 and makes the
//     TMEM round trip of O rare; the true running max is tracked separately for the look-ahead
//     rule.
#pragma once

#include "attn_fwd.cuh"

namespace lamp {

// Self-check build (-DLAMP_SELFCHECK): every index and address is range-checked; a failed
// check records its site in the error word (bits 16..23, reason 0x2) and skips the access.
#ifdef LAMP_SELFCHECK
__device__ __forceinline__ bool lamp_chk(bool ok, uint32_t site) {
  if (!ok) atomicCAS(&g_lamp_error, 0u, 0x2u | (site << 16));
  return ok;
}
#else
__device__ __forceinline__ bool lamp_chk(bool, uint32_t) { return true; }
#endif

struct PPCfg {
  static constexpr int D = 128;
  static constexpr int BN = 128;
  static constexpr int MT = 128;  // rows per query tile (= routing tile)
  static constexpr int Q16_BYTES = MT * D * 2;
  static constexpr int Q8_BYTES = MT * D;
  static constexpr int K8_BYTES = BN * D;        // ring of 8-bit key tiles
  static constexpr int KV_BYTES = BN * D * 2;    // ring of 16-bit key / value tiles
  static constexpr int NS8 = 2;
  static constexpr int NS16 = 3;
  static constexpr int THREADS = 384;            // 2 softmax warpgroups + 1 control warpgroup
  static constexpr int OFF_Q16 = 0;                                // + X * Q16_BYTES
  static constexpr int OFF_Q8 = 2 * Q16_BYTES;                     // + X * Q8_BYTES
  static constexpr int OFF_R8 = OFF_Q8 + 2 * Q8_BYTES;             // + s * K8_BYTES
  static constexpr int OFF_R16 = OFF_R8 + NS8 * K8_BYTES;          // + s * KV_BYTES
  static constexpr int OFF_BAR = OFF_R16 + NS16 * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 512;  // dynamic smem base is 1024-aligned
  static constexpr int TMEM_COLS = 512;
  static constexpr float RESCALE_THRESH = 8.0f;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(OFF_R8 % 1024 == 0 && OFF_R16 % 1024 == 0, "alignment");
};

struct PPBars {
  uint64_t q_full;
  uint64_t q_empty;  // every QK^T MMA of the current work item has completed: Q may be reloaded
  uint64_t full8[PPCfg::NS8], empty8[PPCfg::NS8];
  uint64_t full16[PPCfg::NS16], empty16[PPCfg::NS16];
  uint64_t s_full[2];
  uint64_t s16_full[2];
  uint64_t vote[2];
  uint64_t p_half[2];  // P of keys 0-63 of query tile X is in TMEM
  uint64_t p_full[2];  // all of P of query tile X is in TMEM
  uint64_t o_done[2];
  uint64_t o_free[2];  // the epilogue has read O of query tile X: the next item may overwrite it
  uint64_t drain;
  uint64_t item_full[2];   // the producer has published work item r in slot r & 1
  uint64_t item_empty[2];  // the MMA warp and the 8 softmax warps have read it
  int item[2];             // item index, -1: no item left (or the claim of the counter failed)
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t votes[2][4];
  uint64_t mask[2][2][2];  // [item parity][query tile][word] routing mask (all ones: no mask)
};
static_assert(sizeof(PPBars) <= 512, "barrier block");

struct PPGeo {
  int b, kvh, kt_lo, n;
  int h[2], q0[2], qt[2];  // head, first row and query-tile index of query tile X
  int lo[2], hi[2];        // visible key range (union) of query tile X; lo > hi = none
  int Lq, Lk;              // the sequence's query and key counts
  int q_row0, k_row0;      // its first rows in the Q / O / lse and K / V head planes
  int q_plane[2], kv_plane;  // head planes of query tile X and of the KV head
};

// Work items.  With an even number of query heads per KV head (grouped-query attention) an item
// is one 128-row query tile of two heads of the same KV group: both query tiles see the same
// key tiles, so the two softmax warpgroups stay in step to the item's end, and every K / V tile
// is still loaded once for both.  Otherwise an item is two consecutive query tiles of one head.
// Items are numbered longest-first (causal).
__device__ __forceinline__ bool pp_head_pairs(const AttnParams& p) {
  return ((p.H / p.Hkv) & 1) == 0;
}
__device__ __forceinline__ long long pp_n_items(const AttnParams& p) {
  return pp_head_pairs(p) ? static_cast<long long>(p.B) * (p.H / 2) * p.nqt
                          : static_cast<long long>(p.B) * p.H * ((p.nqt + 1) / 2);
}

// Work distribution (when the KV planes exceed L2; otherwise the fixed order below): a
// launch-wide ticket counter in a scheduler slot (one 64-bit word in
// global memory, 0 when the slot is idle): the launch's tag in the high 32 bits, the next
// ticket in the low 32 bits.  CTA c runs item c first; ticket t gives item gridDim.x + t, so
// that tickets go to whichever CTA asks first and the CTAs' work balances itself whatever the
// items' costs.  Each CTA's producer claims the slot as it starts (idle -> tag, or already
// holding this launch's tag; a slot still held by another launch is waited for, bounded) and
// takes tickets until one is past the last item.  Every CTA takes exactly one such ticket, so
// the CTA that takes ticket n_items - 1 is the last to use the counter: it returns the slot to
// idle, and the next launch given the same slot (a later call, or a replay of a captured
// graph) finds it idle.
constexpr int SCHED_SLOTS = 1024;
__device__ unsigned long long g_lamp_sched[SCHED_SLOTS];

__device__ __forceinline__ bool sched_owned(const AttnParams& p, unsigned long long prev) {
  return prev == 0ull || static_cast<uint32_t>(prev >> 32) == p.sched_tag;
}

__device__ __forceinline__ unsigned long long sched_try_claim(const AttnParams& p) {
  return atomicCAS(p.sched, 0ull, static_cast<unsigned long long>(p.sched_tag) << 32);
}

// The slot held by another launch: wait (bounded) until it is idle and claim it.
__device__ bool sched_claim_wait(const AttnParams& p, const WaitCtx wc) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (sched_owned(p, sched_try_claim(p))) return true;
    __nanosleep(1000);
    if ((it & 7u) == 7u) {
      if (wc.abort && lds_u32(wc.abort)) return false;
      if (globaltimer_ns() - t0 > static_cast<uint64_t>(wc.limit_us) * 1000ull) {
        if (wc.abort) sts_u32(wc.abort, 1u);
        atomicOr(&g_lamp_error, 1u | (W_CLAIM << 8));
        return false;
      }
    }
  }
}

__device__ __forceinline__ int sched_ticket(const AttnParams& p) {
  return static_cast<int>(atomicAdd(p.sched, 1ull) & 0x7FFFFFFFull);
}

// The fixed order (no ticket counter): round r gives CTA c the item r * G + c (r even) or
// r * G + G - 1 - c (r odd), a snake that keeps the CTAs' total work close on the
// longest-first items.  -1: no item left.
__device__ __forceinline__ int pp_item_fixed(const AttnParams& p, int r) {
  const long long n_items = pp_n_items(p);
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const long long j = static_cast<long long>(r) * G + ((r & 1) ? G - 1 - c : c);
  return j < n_items ? static_cast<int>(j) : -1;
}

// With the ticket counter, a consumer warp (all lanes) takes work item r from the producer's
// two-slot ring: the item's index, -1 when none is left, -2 when the wait gave up.
__device__ __forceinline__ int pp_take_item(PPBars& bars, int r, const WaitCtx wc) {
  const int s = r & 1;
  if (!mbar_wait(&bars.item_full[s], static_cast<uint32_t>(r >> 1) & 1u, wc, W_ITEM)) return -2;
  const int item = *reinterpret_cast<volatile int*>(&bars.item[s]);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&bars.item_empty[s]);
  return item;
}

// VARLEN: sequence geometry from the offset arrays (variable-length batches); otherwise the
// dense layout, with every offset a compile-time zero.
// Item order: longest first, all heads side by side; with the ticket counter (TK) the KV planes
// (b * Hkv + kvh) are taken in chunks of p.chunk_kv, so that the K / V tiles the CTAs in flight
// stream stay in L2 while Q and O pass through it, longest first within a chunk.
template <bool VARLEN, bool TK>
__device__ __forceinline__ PPGeo pp_geo(const AttnParams& p, int idx) {
  PPGeo g;
  const int G = p.H / p.Hkv;
  if (!TK && pp_head_pairs(p)) {
    const int BH2 = p.B * (p.H / 2);
    const int qt = p.nqt - 1 - idx / BH2;  // longest-first
    const int bhp = idx - (idx / BH2) * BH2;
    g.b = bhp / (p.H / 2);
    const int hp = bhp - g.b * (p.H / 2);
    for (int x = 0; x < 2; ++x) {
      g.h[x] = 2 * hp + x;
      g.q0[x] = qt * PPCfg::MT;
      g.qt[x] = qt;
    }
  } else if (!TK) {
    const int BH = p.B * p.H;
    const int n_pairs = (p.nqt + 1) / 2;
    const int pair = n_pairs - 1 - idx / BH;  // longest-first
    const int bh = idx - (idx / BH) * BH;
    g.b = bh / p.H;
    for (int x = 0; x < 2; ++x) {
      g.h[x] = bh - g.b * p.H;
      g.q0[x] = (2 * pair + x) * PPCfg::MT;
      g.qt[x] = 2 * pair + x;
    }
  } else if (pp_head_pairs(p)) {
    const int per_qt = p.chunk_kv * (G / 2);  // items of one chunk at one query tile
    const int per_chunk = per_qt * p.nqt;
    const int chunk = idx / per_chunk;
    int rem = idx - chunk * per_chunk;
    const int qr = rem / per_qt;
    rem -= qr * per_qt;
    const int qt = p.nqt - 1 - qr;  // longest-first
    const int kvp = chunk * p.chunk_kv + rem / (G / 2);  // KV plane b * Hkv + kvh
    g.b = kvp / p.Hkv;
    const int hp = (kvp - g.b * p.Hkv) * (G / 2) + (rem - (rem / (G / 2)) * (G / 2));
    for (int x = 0; x < 2; ++x) {
      g.h[x] = 2 * hp + x;
      g.q0[x] = qt * PPCfg::MT;
      g.qt[x] = qt;
    }
  } else {
    const int n_pairs = (p.nqt + 1) / 2;
    const int per_pr = p.chunk_kv * G;  // items of one chunk at one query-tile pair
    const int per_chunk = per_pr * n_pairs;
    const int chunk = idx / per_chunk;
    int rem = idx - chunk * per_chunk;
    const int pr = rem / per_pr;
    rem -= pr * per_pr;
    const int pair = n_pairs - 1 - pr;  // longest-first
    const int kvp = chunk * p.chunk_kv + rem / G;
    g.b = kvp / p.Hkv;
    const int h = (kvp - g.b * p.Hkv) * G + (rem - (rem / G) * G);
    for (int x = 0; x < 2; ++x) {
      g.h[x] = h;
      g.q0[x] = (2 * pair + x) * PPCfg::MT;
      g.qt[x] = 2 * pair + x;
    }
  }
  g.kvh = g.h[0] / (p.H / p.Hkv);
  if (VARLEN) {
    for (int x = 0; x < 2; ++x) {
      const SeqRows sr = seq_rows(p, g.b, g.h[x], g.kvh);
      g.q_plane[x] = sr.q_plane;
      if (x == 0) {
        g.Lq = sr.Lq;
        g.Lk = sr.Lk;
        g.q_row0 = sr.q_row0;
        g.k_row0 = sr.k_row0;
        g.kv_plane = sr.kv_plane;
      }
    }
  } else {
    g.Lq = p.Lq;
    g.Lk = p.Lk;
    g.q_row0 = g.k_row0 = 0;
    g.q_plane[0] = g.b * p.H + g.h[0];
    g.q_plane[1] = g.b * p.H + g.h[1];
    g.kv_plane = g.b * p.Hkv + g.kvh;
  }
  int lo_all = 1 << 30, hi_all = -1;
  for (int x = 0; x < 2; ++x) {
    g.lo[x] = 1;
    g.hi[x] = 0;
    const int r0 = g.q0[x];
    const int r1 = min(g.Lq, r0 + PPCfg::MT) - 1;
    if (r0 > r1) continue;
    int lo0, hi0, lo1, hi1;
    visible_range(p, g.Lq, g.Lk, r0, lo0, hi0);
    visible_range(p, g.Lq, g.Lk, r1, lo1, hi1);
    if (hi1 < 0 || lo0 > hi1) continue;
    g.lo[x] = lo0;
    g.hi[x] = hi1;
    lo_all = min(lo_all, lo0);
    hi_all = max(hi_all, hi1);
  }
  if (hi_all < lo_all) {
    g.kt_lo = 0;
    g.n = 0;
  } else {
    g.kt_lo = lo_all / PPCfg::BN;
    g.n = hi_all / PPCfg::BN - g.kt_lo + 1;
  }
  return g;
}

// Routing mask row of query tile X (W <= 2 words for every supported size), read once.
struct MaskRow {
  uint64_t w0, w1;
};

__device__ __forceinline__ MaskRow load_mask_row(const AttnParams& p, const PPGeo& g, int x) {
  MaskRow m{~0ull, ~0ull};
  const int qt = x ? g.qt[1] : g.qt[0];
  const int hx = x ? g.h[1] : g.h[0];
  if (!p.mask || p.adaptive || qt >= p.nqt) return m;
  const size_t base = (static_cast<size_t>(g.b * p.H + hx) * p.nqt + qt) * p.mask_words;
  if (lamp_chk(base + p.mask_words <= static_cast<size_t>(p.B) * p.H * p.nqt * p.mask_words, 1)) {
    const unsigned long long* mp = reinterpret_cast<const unsigned long long*>(p.mask);
    m.w0 = __ldg(mp + base);
    if (p.mask_words > 1) m.w1 = __ldg(mp + base + 1);
  }
  return m;
}

__device__ __forceinline__ bool tile_live(const PPGeo& g, const AttnParams& p, int x, int kt) {
  const int c0 = kt * PPCfg::BN, c1 = min(g.Lk, c0 + PPCfg::BN) - 1;
  const int lo = x ? g.lo[1] : g.lo[0], hi = x ? g.hi[1] : g.hi[0];
  return lo <= hi && lo <= c1 && hi >= c0;
}

// Key-tile cursor of the producer and MMA warps: the tile's group index advances with the
// tile, so that no integer division sits on the issue path.
struct KtCursor {
  int kt, gi, rem;
};

__device__ __forceinline__ KtCursor kt_first(const AttnParams& p, int kt0) {
  KtCursor c;
  c.kt = kt0;
  c.gi = kt0 / p.group_tiles;
  c.rem = kt0 - c.gi * p.group_tiles;
  return c;
}

__device__ __forceinline__ void kt_next(const AttnParams& p, KtCursor& c) {
  ++c.kt;
  if (++c.rem == p.group_tiles) {
    c.rem = 0;
    ++c.gi;
  }
}

// bitmask routing: true = tiles of routing group gi of this query tile are 16-bit
__device__ __forceinline__ bool group_b16(const AttnParams& p, const MaskRow& m, int gi) {
  if (p.adaptive) return false;
  const uint64_t w = (gi >> 6) ? m.w1 : m.w0;
  return ((w >> (gi & 63)) & 1ull) == 0;
}
// As above, with the mask row of query tile x read from shared memory (it costs the issuing
// warps no registers).
template <class BarsT>
__device__ __forceinline__ bool group_b16(const AttnParams& p, const BarsT& bars, int slot, int x,
                                          int gi) {
  if (p.adaptive) return false;
  const uint64_t w = bars.mask[slot][x][(gi >> 6) & 1];
  return ((w >> (gi & 63)) & 1ull) == 0;
}

// Routing of key tile c.kt for both query tiles.
struct PPPlan {
  bool live0, live1, b16_0, b16_1, need8, need16;
};

template <class BarsT>
__device__ __forceinline__ PPPlan pp_plan(const AttnParams& p, const PPGeo& g, const BarsT& bars,
                                          int slot, const KtCursor& c) {
  PPPlan pl;
  pl.live0 = tile_live(g, p, 0, c.kt);
  pl.live1 = tile_live(g, p, 1, c.kt);
  pl.b16_0 = pl.live0 && group_b16(p, bars, slot, 0, c.gi);
  pl.b16_1 = pl.live1 && group_b16(p, bars, slot, 1, c.gi);
  if (p.adaptive) {
    pl.need8 = pl.need16 = pl.live0 || pl.live1;
  } else {
    pl.need8 = (pl.live0 && !pl.b16_0) || (pl.live1 && !pl.b16_1);
    pl.need16 = pl.b16_0 || pl.b16_1;
  }
  return pl;
}

// ------------------------------------------------------------------ producer ----------

// One lane: for each work item of this CTA, Q16 and Q8 of both query tiles (once the previous
// item's QK^T MMAs have completed) and the item's routing mask rows, then every key tile's K8,
// K16 and V in the MMA warp's order of first use within each ring.  The rings run on across
// items.
template <bool VARLEN, bool TK, class BarsT>
__device__ void pp_producer(const AttnParams& p, uint8_t* smem, BarsT& bars, const WaitCtx wc) {
  using C = PPCfg;
  prefetch_tmap(&p.tm_q16);
  prefetch_tmap(&p.tm_k16);
  prefetch_tmap(&p.tm_v);
  prefetch_tmap(&p.tm_q8);
  prefetch_tmap(&p.tm_k8);
  uint32_t n8 = 0, n16 = 0;
  int pkv = 0, krow0 = 0;  // KV head plane and first key row of the current item's sequence
  auto load8 = [&](int kt) -> bool {
    const int slot = static_cast<int>(n8 % C::NS8);
    const uint32_t use = n8 / C::NS8;
    if (use > 0 && !mbar_wait(&bars.empty8[slot], (use - 1) & 1u, wc, W_EMPTY)) return false;
    mbar_arrive_expect_tx(&bars.full8[slot], C::K8_BYTES);
    tma_load_3d(smem + C::OFF_R8 + slot * C::K8_BYTES, &p.tm_k8, &bars.full8[slot], 0,
                krow0 + kt * C::BN, pkv);
    ++n8;
    return true;
  };
  auto load16 = [&](const CUtensorMap* tm, int kt) -> bool {
    const int slot = static_cast<int>(n16 % C::NS16);
    const uint32_t use = n16 / C::NS16;
    if (use > 0 && !mbar_wait(&bars.empty16[slot], (use - 1) & 1u, wc, W_EMPTY)) return false;
    uint8_t* dst = smem + C::OFF_R16 + slot * C::KV_BYTES;
    mbar_arrive_expect_tx(&bars.full16[slot], C::KV_BYTES);
    tma_load_3d(dst, tm, &bars.full16[slot], 0, krow0 + kt * C::BN, pkv);
    tma_load_3d(dst + C::BN * 128, tm, &bars.full16[slot], 64, krow0 + kt * C::BN, pkv);
    ++n16;
    return true;
  };
  const int n_items = static_cast<int>(pp_n_items(p));
  const int grid = static_cast<int>(gridDim.x);
  // the claim is issued now and its answer read when the first ticket is taken
  const unsigned long long claim0 = TK ? sched_try_claim(p) : 0ull;
  bool claimed = false;
  bool ok = true;
  int next = static_cast<int>(blockIdx.x);  // the first item (the grid never exceeds the items)
  auto take_ticket = [&]() {
    if (!claimed) {
      ok = claimed = sched_owned(p, claim0) || sched_claim_wait(p, wc);
      if (!ok) return;
    }
    next = grid + sched_ticket(p);
  };
  int r = 0;
  for (; ok; ++r) {
    int item;
    if constexpr (TK) {
      // ticket n_items - 1 is the last any CTA takes: return the slot to idle
      if (next == n_items - 1 + grid) atomicExch(p.sched, 0ull);
      // publish item r (or the end) to the consumers
      item = (next < n_items) ? next : -1;
      const int is = r & 1;
      if (r >= 2 && !(ok = mbar_wait(&bars.item_empty[is],
                                     static_cast<uint32_t>((r >> 1) - 1) & 1u, wc, W_ITEM)))
        break;
      bars.item[is] = item;
      mbar_arrive(&bars.item_full[is]);
    } else {
      item = pp_item_fixed(p, r);  // every role computes the fixed order itself
    }
    if (item < 0) break;
    const PPGeo g = pp_geo<VARLEN, TK>(p, item);
    pkv = g.kv_plane;
    krow0 = g.k_row0;
    if (!lamp_chk(g.b * p.H + g.h[1] < p.B * p.H && g.b * p.Hkv + g.kvh < p.B * p.Hkv, 3)) {
      ok = false;
      break;
    }
    if (r > 0 && !(ok = mbar_wait(&bars.q_empty, (r - 1) & 1u, wc, W_EMPTY))) break;
    // the item's mask rows, read by the MMA warp after it has seen this item's Q arrive
    for (int x = 0; x < 2; ++x) {
      const MaskRow m = load_mask_row(p, g, x);
      bars.mask[r & 1][x][0] = m.w0;
      bars.mask[r & 1][x][1] = m.w1;
    }
    mbar_arrive_expect_tx(&bars.q_full, 2 * (C::Q16_BYTES + C::Q8_BYTES));
    for (int x = 0; x < 2; ++x) {
      const int row = g.q_row0 + g.q0[x];
      const int pq = g.q_plane[x];
      for (int c = 0; c < 2; ++c)
        tma_load_3d(smem + C::OFF_Q16 + x * C::Q16_BYTES + c * C::MT * 128, &p.tm_q16,
                    &bars.q_full, c * 64, row, pq);
      tma_load_3d(smem + C::OFF_Q8 + x * C::Q8_BYTES, &p.tm_q8, &bars.q_full, 0, row, pq);
    }
    // The next item's ticket is taken before the loads of the item's second-last key tile,
    // a few key tiles before the CTA is done with the item: late enough that the CTAs which
    // finish first take the next items, early enough that the round trip is over (behind the
    // ring waits of the last two tiles) before the next item is published.
    const int t_ticket = g.n > 2 ? g.n - 2 : 0;
    KtCursor cur = kt_first(p, g.kt_lo);
    for (int t = 0; ok && t < g.n; ++t, kt_next(p, cur)) {
      if (TK && t == t_ticket) {
        take_ticket();
        if (!ok) break;
      }
      const PPPlan pl = pp_plan(p, g, bars, r & 1, cur);
      if (pl.need8 && !(ok = load8(cur.kt))) break;
      if (pl.need16 && !(ok = load16(&p.tm_k16, cur.kt))) break;
      if (!(ok = load16(&p.tm_v, cur.kt))) break;
    }
    if (TK && ok && g.n == 0) take_ticket();
  }
  // Drain: every slot's most recent load must have landed before the CTA may exit.
  const WaitCtx drain{0u, 50000u};  // no abort word: in-flight work always completes
  for (uint32_t it = n8 > static_cast<uint32_t>(C::NS8) ? n8 - C::NS8 : 0; it < n8; ++it)
    mbar_wait(&bars.full8[it % C::NS8], (it / C::NS8) & 1u, drain, W_DRAIN);
  for (uint32_t it = n16 > static_cast<uint32_t>(C::NS16) ? n16 - C::NS16 : 0; it < n16; ++it)
    mbar_wait(&bars.full16[it % C::NS16], (it / C::NS16) & 1u, drain, W_DRAIN);
  if (r > 0) mbar_wait(&bars.q_full, (r - 1) & 1u, drain, W_DRAIN);
}

// ------------------------------------------------------------------ MMA issuer --------

// Run by the whole MMA warp: every lane takes the same waits and computes the same (uniform)
// descriptors; the elected lane issues the MMAs and commits.  Shared-memory descriptors are
// built once per operand region and advanced by constant offsets (16-byte units) per K step.
// Ring cursors (slot, phase) advance in the producer's load order and run on across work
// items; the plan of a key tile is two range tests and two mask bits, with the routing group
// advanced per tile.  Operands of the next key tile are taken before the wait for P, so that
// only MMAs lie between a P tile's arrival and the next QK^T.  Per work item: wait for its Q,
// and before the first QK^T of a query tile for the previous item's epilogue to have read O;
// at the end release Q and publish O.
template <bool BF16, bool ADAPTIVE, bool VARLEN, bool TK>
__device__ void pp_mma(const AttnParams& p, uint8_t* smem, PPBars& bars, uint32_t tbase,
                       const WaitCtx wc) {
  using C = PPCfg;
  const bool leader = elect_one();
  const uint32_t sbase = smem_u32(smem);
  constexpr uint32_t f16 = BF16 ? 1u : 0u;
  constexpr uint32_t id_s16 = idesc(1, f16, f16, 0, 0, C::BN, 128);
  constexpr uint32_t id_s8 = idesc(2, 1, 1, 0, 0, C::BN, 128);  // INT8 only
  constexpr uint32_t id_pv = idesc(1, f16, f16, 0, 1, C::D, 128);
  constexpr bool adaptive = ADAPTIVE;
  // K-major operands: 128-byte rows, 8-row groups 1024 bytes apart; one K step = 32 bytes.
  const uint64_t d_q16 = sdesc(sbase + C::OFF_Q16, 16, 1024, SWZ_128B);
  const uint64_t d_q8 = sdesc(sbase + C::OFF_Q8, 16, 1024, SWZ_128B);
  const uint64_t d_k8 = sdesc(sbase + C::OFF_R8, 16, 1024, SWZ_128B);
  const uint64_t d_k16 = sdesc(sbase + C::OFF_R16, 16, 1024, SWZ_128B);
  // V (MN-major): 64-column atoms BN * 128 bytes apart; one K step = 16 keys = 2048 bytes.
  const uint64_t d_v = sdesc(sbase + C::OFF_R16, C::BN * 128, 1024, SWZ_128B);

  // packed cursors (few registers: this warp's budget is small): bit 0 K8 slot, bit 1 K8 phase,
  // bits 2-3 16-bit slot, bit 4 16-bit phase; bits 8+x vote phase, 10+x P phase, 12+x started,
  // 14+x O of query tile x not yet released by the previous item's epilogue, 16+x O of this
  // item published
  uint32_t st = 0;
  bool ok = true;
  struct Items { int k8, k16; };
  static_assert(C::NS8 == 2 && C::NS16 <= 4, "cursor packing");
  auto take8 = [&]() -> int {
    const int slot = static_cast<int>(st & 1u);
    ok = ok && mbar_wait(&bars.full8[slot], (st >> 1) & 1u, wc, W_FULL);
    st = (slot == C::NS8 - 1) ? ((st & ~1u) ^ 2u) : (st + 1u);
    return slot;
  };
  auto take16 = [&]() -> int {
    const int slot = static_cast<int>((st >> 2) & 3u);
    ok = ok && mbar_wait(&bars.full16[slot], (st >> 4) & 1u, wc, W_FULL);
    st = (slot == C::NS16 - 1) ? ((st & ~12u) ^ 16u) : (st + 4u);
    return slot;
  };
  auto live = [](uint32_t pl, int x) { return (pl >> x) & 1u; };
  auto b16 = [](uint32_t pl, int x) { return ((pl >> (2 + x)) & 1u) != 0; };
  auto take_k = [&](uint32_t pl, Items& it) {
    it.k8 = (pl & 16u) ? take8() : -1;
    it.k16 = (pl & 32u) ? take16() : -1;
    tc_fence_after();
  };
  auto issue_s = [&](int x, bool sixteen, int slot) {
    const uint32_t dS = tbase + static_cast<uint32_t>(x * C::BN);
    if (sixteen) {
      if (!lamp_chk(slot >= 0 && slot < C::NS16, 5)) return;
      const uint64_t qa = d_q16 + static_cast<uint64_t>(x * (C::Q16_BYTES >> 4));
      const uint64_t kb = d_k16 + static_cast<uint64_t>(slot * (C::KV_BYTES >> 4));
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::D / 16; ++s) {
          const uint64_t off = static_cast<uint64_t>((s >> 2) * ((C::MT * 128) >> 4) + (s & 3) * 2);
          mma_f16_ss(dS, qa + off, kb + off, id_s16, s > 0 ? 1u : 0u);
        }
      }
    } else {
      if (!lamp_chk(slot >= 0 && slot < C::NS8, 5)) return;
      const uint64_t qa = d_q8 + static_cast<uint64_t>(x * (C::Q8_BYTES >> 4));
      const uint64_t kb = d_k8 + static_cast<uint64_t>(slot * (C::K8_BYTES >> 4));
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::D / 32; ++s)
          mma_i8_ss(dS, qa + static_cast<uint64_t>(s * 2), kb + static_cast<uint64_t>(s * 2), id_s8,
                    s > 0 ? 1u : 0u);
      }
    }
  };
  auto commit = [&](uint64_t* bar) {
    if (leader) tc_commit(bar);
  };
  // the previous item's epilogue must have read O of query tile x (phase r - 1 of o_free) before
  // this item's first P.V overwrites it
  auto o_released = [&](int x, int r) {
    if ((st >> (14 + x)) & 1u) {
      ok = ok && mbar_wait(&bars.o_free[x], (r - 1) & 1u, wc, W_ODONE);
      st &= ~(1u << (14 + x));
    }
  };
  auto first_s = [&](int x, bool b16x, const Items& it) {
    const bool sixteen = !adaptive && b16x;
    issue_s(x, sixteen, sixteen ? it.k16 : it.k8);
    commit(&bars.s_full[x]);
  };
  // P.V over keys [64 * half, 64 * half + 64) of the tile; P (16-bit pairs) sits in columns
  // 0-63 of S_X, keys 0-63 in columns 0-31
  auto pv = [&](int x, int vslot, int half, bool acc) {
    const uint64_t vb = d_v + static_cast<uint64_t>(vslot * (C::KV_BYTES >> 4));
    const uint32_t pt = tbase + static_cast<uint32_t>(x * C::BN);
    const uint32_t ot = tbase + static_cast<uint32_t>(2 * C::BN + x * C::D);
    if (leader) {
#pragma unroll
      for (int s = 4 * half; s < 4 * half + 4; ++s)
        mma_f16_ts(ot, pt + s * 8, vb + static_cast<uint64_t>(s * ((16 * 128) >> 4)), id_pv,
                   (acc || s > 0) ? 1u : 0u);
    }
  };

  for (int r = 0; ok; ++r) {
    const int item = TK ? pp_take_item(bars, r, wc) : pp_item_fixed(p, r);
    if (item < 0) break;
    const PPGeo g = pp_geo<VARLEN, TK>(p, item);
    const int ms = r & 1;  // mask slot of this item
    const int ra0 = (g.lo[0] <= g.hi[0]) ? g.lo[0] / C::BN : (1 << 30);
    const int rb0 = (g.lo[0] <= g.hi[0]) ? g.hi[0] / C::BN : -1;
    const int ra1 = (g.lo[1] <= g.hi[1]) ? g.lo[1] / C::BN : (1 << 30);
    const int rb1 = (g.lo[1] <= g.hi[1]) ? g.hi[1] / C::BN : -1;
    // plan bits: 1 live0, 2 live1, 4 b16_0, 8 b16_1, 16 need8, 32 need16
    auto plan = [&](int kt, int gi) -> uint32_t {
      const bool l0 = kt >= ra0 && kt <= rb0, l1 = kt >= ra1 && kt <= rb1;
      const bool h0 = l0 && group_b16(p, bars, ms, 0, gi), h1 = l1 && group_b16(p, bars, ms, 1, gi);
      const bool n8 = adaptive ? (l0 || l1) : ((l0 && !h0) || (l1 && !h1));
      const bool n16 = adaptive ? (l0 || l1) : (h0 || h1);
      return (l0 ? 1u : 0u) | (l1 ? 2u : 0u) | (h0 ? 4u : 0u) | (h1 ? 8u : 0u) | (n8 ? 16u : 0u) |
             (n16 ? 32u : 0u);
    };
    if (!(ok = mbar_wait(&bars.q_full, ms, wc, W_QFULL))) break;
    tc_fence_after();
    st &= ~((3u << 12) | (3u << 16));  // no P.V of this item yet, O not published
    if (r > 0) st |= 3u << 14;         // O of both tiles held by the previous item's epilogue

    Items cur{-1, -1}, nxt{-1, -1};
    int kt = g.kt_lo;
    int gi = kt / p.group_tiles, grem = kt - gi * p.group_tiles;
    uint32_t pl = plan(kt, gi);
    if (g.n > 0) {
      take_k(pl, cur);
      if (ok && live(pl, 0)) first_s(0, b16(pl, 0), cur);
      if (ok && live(pl, 1)) first_s(1, b16(pl, 1), cur);
    }
    const int kt_end = g.kt_lo + g.n;
    for (; ok && kt < kt_end; ++kt) {
      const bool has_next = kt + 1 < kt_end;
      if (++grem == p.group_tiles) {
        grem = 0;
        ++gi;
      }
      const uint32_t pn = has_next ? plan(kt + 1, gi) : 0u;
      if (adaptive) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (!ok || !live(pl, x)) continue;
          if (!(ok = mbar_wait(&bars.vote[x], (st >> (8 + x)) & 1u, wc, W_VOTE))) break;
          st ^= 1u << (8 + x);
          tc_fence_after();
          const volatile uint32_t* vv = bars.votes[x];
          uint32_t any = 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) any |= vv[w];
          if (any) {
            issue_s(x, true, cur.k16);
            commit(&bars.s16_full[x]);
          }
        }
        if (!ok) break;
      }
      // every QK^T MMA of this key tile has been issued: release its K slots when they finish,
      // and Q once the item's last key tile is reached
      if (cur.k8 >= 0) commit(&bars.empty8[cur.k8]);
      if (cur.k16 >= 0) commit(&bars.empty16[cur.k16]);
      if (!has_next) commit(&bars.q_empty);
      // V of this tile and K of the next were loaded long ago: take them before waiting for P
      const int vslot = take16();
      if (has_next) take_k(pn, nxt);
      tc_fence_after();
      if (!ok) break;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (!ok) break;
        if (live(pl, x)) {
          const uint32_t cp = (st >> (10 + x)) & 1u;
          // the first half of P is published while the softmax exponentiates the second
          const bool started = ((st >> (12 + x)) & 1u) != 0;
          if (!started) o_released(x, r);
          if (!(ok = ok && mbar_wait(&bars.p_half[x], cp, wc, W_PFULL))) break;
          tc_fence_after();
          pv(x, vslot, 0, started);
          if (!(ok = mbar_wait(&bars.p_full[x], cp, wc, W_PFULL))) break;
          tc_fence_after();
          pv(x, vslot, 1, true);
          st = (st ^ (1u << (10 + x))) | (1u << (12 + x));
          if (!(has_next && live(pn, x))) {  // the query tile's last key tile: publish O
            commit(&bars.o_done[x]);
            st |= 1u << (16 + x);
          }
        }
        if (has_next && live(pn, x)) first_s(x, b16(pn, x), nxt);
      }
      if (!ok) break;
      commit(&bars.empty16[vslot]);
      cur = nxt;
      pl = pn;
    }
    if (!ok) break;
    if (g.n == 0) commit(&bars.q_empty);
    for (int x = 0; x < 2; ++x) {  // a query tile without a visible key tile: O is zero
      if (!((st >> (16 + x)) & 1u)) {
        o_released(x, r);
        commit(&bars.o_done[x]);
      }
    }
  }
  commit(&bars.drain);
  const WaitCtx drain{0u, 50000u};  // no abort word: in-flight work always completes
  mbar_wait(&bars.drain, 0, drain, W_DRAIN);
}

// ------------------------------------------------------------------ softmax -----------

// (f32x2 helpers, max3 and the mixed-precision adds come from attn_fwd.cuh)

// A thread owns row r of query tile X.  Per key tile: read the row of S from TMEM, turn it
// into fp32 values of the raw product (exact int32 -> fp32 for 8-bit tiles), mask, take the
// row max, vote (look-ahead rule), exponentiate against the lazy reference max, pack P as
// 16-bit pairs into the row's S columns 0-63 (each 32-column chunk stored as soon as it is
// ready), and keep two row sums: of the exact p (for lse) and of the rounded p that the P.V
// MMA multiplies (for O).
//
// The warpgroup's first warp also issues its query tile's MMAs (the elected lane issues; all
// lanes keep the same, warp-uniform ring state): as soon as the whole P tile is in TMEM it
// issues P.V and the next key tile's QK^T, so that no other warp stands between a finished P
// and the tensor core.  Both warpgroups take every key tile's ring slots in the producer's
// order (passing the tiles their query tile does not see) and release each slot with a
// commit: a slot is free once both have released it.
// One work item of the softmax role (it = the CTA's item count, the parity of its per-item
// barrier phases).  The phase counters of the per-tile barriers run on across items.  Returns
// false when a wait gave up.
template <bool BF16, bool ADAPTIVE, bool VARLEN, bool DBG>
__device__ __forceinline__ bool pp_softmax_item(const AttnParams& p, const PPGeo& g, PPBars& bars,
                                                uint32_t tbase, const WaitCtx wc, int it,
                                                uint32_t& cs, uint32_t& c16, uint32_t& cvv,
                                                uint32_t (&raw)[PPCfg::BN]) {
  using C = PPCfg;
  constexpr int N = C::BN;
  const int warp = threadIdx.x >> 5;
  const int x = warp >> 2;                  // query tile of this warpgroup
  const int q4 = warp & 3;                  // TMEM lane quadrant
  const int lane = threadIdx.x & 31;
  const int r = q4 * 32 + lane;
  const int i = (x ? g.q0[1] : g.q0[0]) + r;
  const bool row_valid = i < g.Lq;
  const int qt = x ? g.qt[1] : g.qt[0];
  const int bh_q = g.b * p.H + (x ? g.h[1] : g.h[0]);
  const uint32_t lane_base = tbase + (static_cast<uint32_t>(q4 * 32) << 16);
  const uint32_t s_col = static_cast<uint32_t>(x * C::BN);
  const uint32_t o_col = static_cast<uint32_t>(2 * C::BN + x * C::D);
  int lo_r = 1, hi_r = 0;
  if (row_valid) visible_range(p, g.Lq, g.Lk, i, lo_r, hi_r);
  const float sq = (row_valid && qt < p.nqt) ? __ldg(p.q_scale + static_cast<size_t>(bh_q) * p.nqt + qt) : 0.0f;
  const float* ks_row = p.k_scale + static_cast<size_t>(g.b * p.Hkv + g.kvh) * p.nkt;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float sq_scale = sq * p.scale_log2;
  const MaskRow mrow = load_mask_row(p, g, x);

  float m_ref = NEG_INF;   // max used for the exponentials (lazy)
  float m_true = NEG_INF;  // true running max of the used scores (look-ahead rule)
  float l_ex = 0.0f, l_rd = 0.0f;
  bool ok = true, any_pv = false;

  auto load_s = [&]() {
#pragma unroll
    for (int c = 0; c < N / 32; ++c)
      tmem_ld32(lane_base + s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
    tmem_wait_ld();
  };
  // int32 accumulators -> fp32, exact (|acc| < 2^22)
  auto int_to_float = [&]() {
#pragma unroll
    for (int c = 0; c < N; ++c) raw[c] = __float_as_uint(static_cast<float>(static_cast<int>(raw[c])));
  };
  // keep columns [a, b] of the tile (the row's visible keys), -inf elsewhere; branch-free
  auto apply_mask = [&](int j0) {
    const int a = row_valid ? lo_r - j0 : N;
    const int b = row_valid ? hi_r - j0 : -1;
#pragma unroll
    for (int c = 0; c < N; ++c) raw[c] = (c < a || c > b) ? 0xff800000u : raw[c];
  };
  auto raw_max = [&]() -> float {
    float m0 = NEG_INF, m1 = NEG_INF, m2 = NEG_INF, m3 = NEG_INF;
#pragma unroll
    for (int c = 0; c < N; c += 8) {
      m0 = max3(m0, __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
      m1 = max3(m1, __uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3]));
      m2 = max3(m2, __uint_as_float(raw[c + 4]), __uint_as_float(raw[c + 5]));
      m3 = max3(m3, __uint_as_float(raw[c + 6]), __uint_as_float(raw[c + 7]));
    }
    return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  };

  // The live key tiles of query tile X form one range [kt_first, kt_last] (causal and window
  // limits are monotone in the row); the K scale of the next tile is fetched one tile ahead
  // and the tile's routing group advances with it.
  const int lo_x = x ? g.lo[1] : g.lo[0], hi_x = x ? g.hi[1] : g.hi[0];
  const int kt_first = (lo_x <= hi_x) ? lo_x / N : 1, kt_last = (lo_x <= hi_x) ? hi_x / N : 0;
  float ks_n = (kt_first <= kt_last) ? __ldg(ks_row + kt_first) : 0.0f;
  int gi = kt_first / p.group_tiles, grem = kt_first - gi * p.group_tiles;

  for (int kt = kt_first; ok && kt <= kt_last; ++kt) {
    const float ks = ks_n;
    if (kt < kt_last) ks_n = __ldg(ks_row + kt + 1);
    const int gcur = gi;
    if (++grem == p.group_tiles) {
      grem = 0;
      ++gi;
    }

    if (!(ok = warp_wait(&bars.s_full[x], cs & 1u, wc, W_SFULL))) break;
    ++cs;
    tc_fence_after();
    load_s();
    const int j0 = kt * N;
    const bool full = row_valid && j0 >= lo_r && j0 + N - 1 <= hi_r;
    bool sixteen = !ADAPTIVE && group_b16(p, mrow, gcur);
    if constexpr (DBG)  // debug capture of the raw S this row read (capture build only)
      dbg_dump<N>(p, sixteen ? p.dbg_s16 : p.dbg_s8, C::MT, N, bh_q, qt, kt, r, 0, raw);
    // (a zero block scale would turn masked -inf entries into NaN: keep it positive; the
    // scores of an all-zero block are 0 either way)
    float cscale = sixteen ? p.scale_log2 : fmaxf(sq_scale * ks, 1e-30f);
    if (!sixteen) int_to_float();
    if (!full) apply_mask(j0);
    float tmax = raw_max();
    bool flagged = false;
    if (ADAPTIVE) {
      const float t8 = (tmax == NEG_INF) ? NEG_INF : tmax * cscale;
      const bool vote = (t8 != NEG_INF) && (t8 >= m_true - p.tau_log2);
      const uint32_t wv = __any_sync(0xFFFFFFFFu, vote) ? 1u : 0u;
      if (lane == 0) bars.votes[x][q4] = wv;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.vote[x]);
      if (!(ok = warp_wait(&bars.vote[x], cvv & 1u, wc, W_VOTE))) break;
      ++cvv;
      const volatile uint32_t* vv = bars.votes[x];
      flagged = (vv[0] | vv[1] | vv[2] | vv[3]) != 0;
      if (flagged) {
        if (!(ok = warp_wait(&bars.s16_full[x], c16 & 1u, wc, W_S16))) break;
        ++c16;
        tc_fence_after();
        load_s();
        if constexpr (DBG) dbg_dump<N>(p, p.dbg_s16, C::MT, N, bh_q, qt, kt, r, 0, raw);
        sixteen = true;
        cscale = p.scale_log2;
        if (!full) apply_mask(j0);
        tmax = raw_max();
      }
    }
    if (p.route && q4 == 0 && lane == 0 &&
        lamp_chk((static_cast<size_t>(bh_q) * p.nqt + qt) * p.nkt + kt <
                     static_cast<size_t>(p.B) * p.H * p.nqt * p.nkt && qt < p.nqt, 11))
      p.route[(static_cast<size_t>(bh_q) * p.nqt + qt) * p.nkt + kt] =
          ADAPTIVE ? (flagged ? 3 : 1) : (sixteen ? 2 : 1);

    const float tl = (tmax == NEG_INF) ? NEG_INF : tmax * cscale;  // log2 units
    m_true = fmaxf(m_true, tl);
    // lazy reference max: moves only when the row max exceeds it by more than the threshold
    const bool move = (tl != NEG_INF) && (m_ref == NEG_INF || tl > m_ref + C::RESCALE_THRESH);
    const float new_ref = move ? tl : m_ref;
    const float alpha = move ? ((m_ref == NEG_INF) ? 0.0f : ex2(m_ref - new_ref)) : 1.0f;
    if (any_pv && __any_sync(0xFFFFFFFFu, move && m_ref != NEG_INF)) {
      // P.V of this row's previous tile has completed (this S was issued after it)
      const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
      for (int c = 0; c < C::D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(lane_base + o_col + c * 32, ov);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float lo, hi;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), a2, 0ull),
                    lo, hi);
          ov[e] = __float_as_uint(lo);
          ov[e + 1] = __float_as_uint(hi);
        }
        tmem_st16(lane_base + o_col + c * 32, ov);
        tmem_st16(lane_base + o_col + c * 32 + 16, ov + 16);
      }
      tmem_wait_st();
    }
    l_ex *= alpha;
    l_rd *= alpha;
    m_ref = new_ref;

    // p = 2^(value * cscale - m_ref); masked entries hold -inf and give 0.  Each 32-column
    // chunk of P (16 packed columns) is stored as soon as it is ready.
    const float mu = (m_ref == NEG_INF) ? 0.0f : m_ref;
    const uint64_t c2 = f2_pack(cscale, cscale);
    const uint64_t nb2 = f2_pack(-mu, -mu);
    uint64_t se0 = 0, se1 = 0;
    float sr0 = 0.f, sr1 = 0.f, sr2 = 0.f, sr3 = 0.f;
#pragma unroll
    for (int c = 0; c < N; c += 2) {
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), c2, nb2),
                x0, x1);
      float p0, p1;
      p0 = ex2(x0); p1 = ex2(x1);
      uint32_t pk;
      if (BF16) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk = *reinterpret_cast<uint32_t*>(&h2);
      } else {
        __half2 h2 = __floats2half2_rn(p0, p1);
        pk = *reinterpret_cast<uint32_t*>(&h2);
      }
      if (c & 2) {
        se1 = f2_add(se1, f2_pack(p0, p1));
        sr2 = add_lo16<BF16>(sr2, pk);
        sr3 = add_hi16<BF16>(sr3, pk);
      } else {
        se0 = f2_add(se0, f2_pack(p0, p1));
        sr0 = add_lo16<BF16>(sr0, pk);
        sr1 = add_hi16<BF16>(sr1, pk);
      }
      raw[c >> 1] = pk;
      if (c == 94) {
        // P of keys 0-63 (stored with the chunks of columns 0-63) is in TMEM: publish it, so
        // that the first half of P.V overlaps the exponentials of the second half
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_half[x]);
      }
      if ((c & 31) == 30) tmem_st16(lane_base + s_col + (c >> 5) * 16, &raw[(c >> 5) * 16]);
    }
    {
      float a0, a1;
      f2_unpack(f2_add(se0, se1), a0, a1);
      l_ex += a0 + a1;
      l_rd += (sr0 + sr1) + (sr2 + sr3);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.p_full[x]);
    any_pv = true;
  }
  if (!ok) return false;

  // epilogue: O / l and lse.  O is read from TMEM in one go and released at once, so that the
  // next item's P.V may start while this one is normalised and stored.
  if (!warp_wait(&bars.o_done[x], it & 1, wc, W_ODONE)) return false;
  tc_fence_after();
  if (any_pv) {
#pragma unroll
    for (int c = 0; c < C::D / 32; ++c)
      tmem_ld32(lane_base + o_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
    tmem_wait_ld();
  } else {
#pragma unroll
    for (int e = 0; e < C::D; ++e) raw[e] = 0u;
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&bars.o_free[x]);
  const float inv = (l_rd > 0.0f) ? 1.0f / l_rd : 0.0f;
  const int pq = x ? g.q_plane[1] : g.q_plane[0];
  const size_t orow = (static_cast<size_t>(pq) * p.q_rows + g.q_row0 + (row_valid ? i : 0)) * C::D;
  if (row_valid &&
      lamp_chk(orow + C::D <= static_cast<size_t>(p.cu_q ? p.H : p.B * p.H) * p.q_rows * C::D, 12)) {
    // 32-byte stores: each thread writes whole sectors of its row
    auto sc = [&](int e) { return __float_as_uint(__uint_as_float(raw[e]) * inv); };
    if (p.out_f32) {
      float* dst = static_cast<float*>(p.o) + orow;
#pragma unroll
      for (int e = 0; e < C::D; e += 8)
        st_global_v8(dst + e, sc(e), sc(e + 1), sc(e + 2), sc(e + 3), sc(e + 4), sc(e + 5), sc(e + 6),
                     sc(e + 7));
    } else {
      uint16_t* dst = static_cast<uint16_t*>(p.o) + orow;
#pragma unroll
      for (int e = 0; e < C::D; e += 16) {
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float a = __uint_as_float(raw[e + 2 * q]) * inv;
          const float b2 = __uint_as_float(raw[e + 2 * q + 1]) * inv;
          if (BF16) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(a, b2);
            w[q] = *reinterpret_cast<uint32_t*>(&v2);
          } else {
            __half2 v2 = __floats2half2_rn(a, b2);
            w[q] = *reinterpret_cast<uint32_t*>(&v2);
          }
        }
        st_global_v8(dst + e, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
      }
    }
  }
  if (row_valid && p.lse)
    p.lse[static_cast<size_t>(pq) * p.q_rows + g.q_row0 + i] =
        (l_ex > 0.0f) ? m_ref * 0.69314718055994530942f + logf(l_ex) : NEG_INF;
  return true;
}

// The softmax role: the CTA's work items in turn.
template <bool BF16, bool ADAPTIVE, bool VARLEN, bool DBG, bool TK>
__device__ void pp_softmax(const AttnParams& p, PPBars& bars, uint32_t tbase, const WaitCtx wc) {
  uint32_t cs = 0, c16 = 0, cvv = 0;
  uint32_t raw[PPCfg::BN];
  for (int it = 0;; ++it) {
    const int item = TK ? pp_take_item(bars, it, wc) : pp_item_fixed(p, it);
    if (item < 0) break;
    const PPGeo g = pp_geo<VARLEN, TK>(p, item);
    if (!pp_softmax_item<BF16, ADAPTIVE, VARLEN, DBG>(p, g, bars, tbase, wc, it, cs, c16, cvv, raw)) break;
  }
}

// ------------------------------------------------------------------ kernel ------------

template <bool BF16, bool ADAPTIVE, bool VARLEN, bool DBG, bool TK>
__global__ void __launch_bounds__(PPCfg::THREADS, 1)
    attn_fwd_pp_kernel(const __grid_constant__ AttnParams p) {
  using C = PPCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the layouts need a 1024-aligned base
    if (threadIdx.x == 0) atomicOr(&g_lamp_error, 0x4u);
    return;
  }
  PPBars& bars = *reinterpret_cast<PPBars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < C::NS8; ++s) {
      mbar_init(&bars.full8[s], 1);
      mbar_init(&bars.empty8[s], 1);
    }
    for (int s = 0; s < C::NS16; ++s) {
      mbar_init(&bars.full16[s], 1);
      mbar_init(&bars.empty16[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.s16_full[x], 1);
      mbar_init(&bars.vote[x], 4);
      mbar_init(&bars.p_half[x], 4);
      mbar_init(&bars.p_full[x], 4);
      mbar_init(&bars.o_done[x], 1);
      mbar_init(&bars.o_free[x], 4);
    }
    mbar_init(&bars.drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.item_full[i], 1);
      mbar_init(&bars.item_empty[i], 9);  // the MMA warp and the 8 softmax warps
    }
    bars.abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;
  const WaitCtx wc{smem_u32(&bars.abort), static_cast<uint32_t>(p.wait_ns / 1000)};
  // Register split within the launch allotment of 384 x 168: the control warpgroup gives
  // back to 104 per thread, the two softmax warpgroups grow to 200
  // (128 * 104 + 256 * 200 = 64512 = 384 * 168).
  // Every role derives each item's geometry itself; with the ticket counter the producer
  // takes the tickets and publishes each item to the other roles.
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    pp_softmax<BF16, ADAPTIVE, VARLEN, DBG, TK>(p, bars, tbase, wc);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory");
    if (warp == 8) {
      if ((threadIdx.x & 31) == 0) pp_producer<VARLEN, TK>(p, smem, bars, wc);
    } else if (warp == 9) {
      pp_mma<BF16, ADAPTIVE, VARLEN, TK>(p, smem, bars, tbase, wc);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace lamp
