// Routed mixed-precision attention forward for sm_100a.
//
// What it computes (TileMix page, section 2 "How It Works"; LampAttention abstract):
// softmax(scale * Q K^T) V over the visible (causal / sliding-window) pairs, where each score
// tile (routing tile BM x BN) is either the 8-bit product of per-block quantised Q and K,
// rescaled by the two block scales, or the 16-bit product of the inputs.  The choice comes from
// a packed bitmask (one bit per group of key tiles, 0 = 16-bit) or from the look-ahead rule
// (recompute in 16 bits when some row's 8-bit tile max reaches the running row max minus tau).
// Both paths update one online-softmax state (m, l) per row; P.V is 16-bit.
//
// B200 design:
//   * one CTA per (batch, head, 128-row query tile); grid ordered longest-first (causal);
//     variable-length batches (TileMix page, section 4) take each sequence's lengths and first
//     rows from offset arrays and address packed [heads][rows][D] tensors;
//   * warp 8 (one thread) streams Q16/Q8 once and then K8 / K16 / V tiles with TMA into a
//     ring of shared-memory slots (128-byte or 64-byte swizzled, the layouts the tensor core
//     reads), each slot guarded by full/empty mbarriers;
//   * warp 9 issues tcgen05 MMAs (the whole warp runs the loop, one elected lane issues):
//     S = Q8 K8^T (kind::i8 into int32 TMEM or kind::f8f6f4 into fp32 TMEM), S = Q16 K16^T
//     (kind::f16), O += P V with P read from TMEM; the S buffer is double-buffered so S(t+1)
//     runs on the tensor core while rows of S(t) are in the softmax;
//   * warps 0-7 own one query row per two threads (TMEM lane = row; warps 0-3 columns 0..BN/2,
//     warps 4-7 the rest): they read S from TMEM, dequantise, mask, exchange the half-row
//     maxima, vote on the look-ahead rule, run the online softmax (MUFU ex2, lazy reference
//     max), store P as packed 16-bit pairs into the S columns, rescale O in TMEM when the
//     reference moves, and write O / lse at the end;
//   * routing tiles of 64 query rows (D = 64, 256) are stacked two per 128-row MMA;
//   * a two-phase key tile (look-ahead mode, or stacked halves of different precisions) has
//     an 8-bit and a 16-bit S.  At D = 64 and 128 the 16-bit S has TMEM columns of its own and
//     is issued right behind the 8-bit one (in look-ahead mode speculatively: the rows read it
//     only when the vote flags the tile, and the tile's result is the same as if it had been
//     issued after the vote); at D = 256 it goes into the 8-bit S's columns once every row has
//     read its 8-bit scores.
// Every mbarrier wait is bounded; on a timeout the CTA records the failure, stops, drains its
// in-flight copies and MMAs, frees its TMEM and exits.
#pragma once

#include <cuda.h>

#include <cstdint>

#include "ptx.cuh"

namespace lamp {


// where-codes recorded with a timeout (bits 8..15 of the error word)
enum : uint32_t {
  W_QFULL = 1, W_EMPTY = 2, W_FULL = 3, W_SFULL = 4, W_S16 = 5, W_VOTE = 6, W_PFULL = 7,
  W_ODONE = 8, W_DRAIN = 9, W_SELFTEST = 10, W_XCH = 11, W_ZFREE = 12, W_OSTAGE = 13,
  W_ITEM = 14, W_CLAIM = 15
};

struct AttnParams {
  CUtensorMap tm_q16;  // [B*H][Lq][D] 16-bit, box 64 x 128 x 1, 128B swizzle
  CUtensorMap tm_k16;  // [B*Hkv][Lk][D] 16-bit, box 64 x BN x 1, 128B swizzle
  CUtensorMap tm_v;    // [B*Hkv][Lk][D] 16-bit, box 64 x BN x 1, 128B swizzle
  CUtensorMap tm_q8;   // [B*H][Lq][D] 8-bit, box min(D,128) x 128 x 1
  CUtensorMap tm_k8;   // [B*Hkv][Lk][D] 8-bit, box min(D,128) x BN x 1
  // 8-bit P.V mode: V in E4M3, channel-major [B*Hkv][D][Lk rounded up to 16], box BN x D x 1,
  // 128B swizzle, and its per-channel scales [B*Hkv][D]
  CUtensorMap tm_v8;
  const float* v_scale;
  const float* q_scale;  // [B][H][nQT]
  const float* k_scale;  // [B][Hkv][nKT]
  const uint64_t* mask;  // [B][H][nQT][W] or null
  void* o;
  float* lse;
  uint8_t* route;
  int B, H, Hkv, Lq, Lk;  // variable-length batches: Lq, Lk = the longest sequence
  int n_ct, nqt, nkt, mask_words, group_tiles;
  // variable-length batches: row offsets [B + 1] of the sequences in the packed [heads][rows][D]
  // tensors (null: dense [B][heads][L][D]); q_rows = rows per head plane of Q, O and lse
  const int* cu_q;
  const int* cu_k;
  int q_rows, k_rows;
  int causal, window;
  float scale_log2, tau_log2;
  float skip_log2;  // look-ahead mode: drop a tile every row of which is this far below its
                    // running max (log2 units; +inf: never)
  int adaptive, e4m3, bf16, out_f32;
  // KV planes (b * Hkv + kvh) per chunk of the CTA / work-item order (a divisor of B * Hkv):
  // the work of one chunk runs before the next chunk's, longest query tiles first
  int chunk_kv;
  // two-tile kernel: its scheduler slot (work-item ticket counter) and the launch's nonzero tag
  unsigned long long* sched;
  uint32_t sched_tag;
  uint64_t wait_ns;
  // Debug capture (lamp_attn_debug only; unused elsewhere): slot map [B][H][nQT][nKT] (slot of
  // a routing tile, < 0 = not captured), and the raw score tiles [slots][BM][BN]: the 8-bit
  // product words as read from TMEM (int32 or fp32 bits) and the 16-bit product (fp32).
  const int* dbg_slot;
  uint32_t* dbg_s8;
  uint32_t* dbg_s16;
  int dbg_nslots;
};

template <int D_, int BN_, bool STACK_, bool PV8_ = false>
struct AttnCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;
  static constexpr bool STACK = STACK_;        // routing tiles of 64 rows, two per MMA tile
  // 8-bit exponentials and 8-bit P.V: P goes to shared memory in E4M3 (one 16 KB buffer per S
  // buffer) and P.V is the SS-form E4M3 MMA with V channel-major in the ring
  static constexpr bool PV8 = PV8_;
  static constexpr int BM = STACK ? 64 : 128;  // routing tile rows
  static constexpr int MT = 128;               // MMA tile rows
  static constexpr int Q16_BYTES = MT * D * 2;
  static constexpr int Q8_BYTES = MT * D;
  static constexpr int SLOT_BYTES = BN * D * 2;
  static constexpr int NS = PV8 ? 4 : (D == 64) ? 8 : (D == 128 ? 5 : 2);
  static constexpr bool Q8_SW64 = (D == 64);  // 64-byte rows of 8-bit codes
  static constexpr int C16 = D / 64;           // 128-byte chunks of a 16-bit row
  static constexpr int C8 = (D == 64) ? 1 : D / 128;
  static constexpr int TMEM_O = 2 * BN;
  // A separate TMEM region Z for the 16-bit S of two-phase key tiles, where the columns allow
  // (D = 64, 128): the 16-bit MMA is then issued right behind the 8-bit one instead of after
  // every row has read the 8-bit scores.  At D = 256 (S x 2 + O fill all 512 columns) the
  // 16-bit S goes into the 8-bit S's own columns after the rows have read them.
  static constexpr bool SEP16 = 3 * BN + D <= 512;
  static constexpr int TMEM_Z = 2 * BN + D;
  static constexpr int TMEM_COLS = ((SEP16 ? 3 * BN : 2 * BN) + D) <= 256 ? 256 : 512;
  static constexpr int OFF_Q16 = 0;
  static constexpr int OFF_Q8 = Q16_BYTES;
  static constexpr int OFF_SLOTS = Q16_BYTES + Q8_BYTES;
  static constexpr int OFF_P8 = OFF_SLOTS + NS * SLOT_BYTES;  // [2][MT rows][BN bytes], PV8
  static constexpr int P8_BYTES = MT * BN;
  static constexpr int OFF_BAR = OFF_P8 + (PV8 ? 2 * P8_BYTES : 0);
  static constexpr int BAR_BYTES = 512;
  static constexpr int OFF_XCH = OFF_BAR + BAR_BYTES;  // row-pair exchange: float [2][2][MT]
  static constexpr int SMEM_BYTES = OFF_XCH + 2 * 2 * MT * 4;  // dynamic base is 1024-aligned
  static constexpr int THREADS = 320;  // 8 softmax warps (two per row), producer, MMA
  static_assert(OFF_Q8 % 1024 == 0 && OFF_SLOTS % 1024 == 0 && SLOT_BYTES % 1024 == 0, "align");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(2 * BN + D <= 512, "tmem");
  static_assert(D != 256 || MT * D * 4 <= OFF_BAR, "O staging");
  static_assert(!PV8 || (D == 128 && BN == 128 && !STACK), "8-bit P.V: D = 128, one routing tile");
};

struct Bars {
  uint64_t q_full;
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t s_full[2];
  uint64_t s16_full[2];
  uint64_t vote[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint64_t z_free;   // the rows have finished with the 16-bit S region Z (8 warp arrivals)
  uint64_t o_final;  // every P.V of the CTA has completed (one phase)
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t votes[2][8];
  uint64_t xbar[4];  // row-pair exchange of lane quadrant q (64 arrivals)
  uint64_t ostage;   // every softmax warp has put its rows of O into the staging area (8)
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// Per-key-tile routing plan, computed identically by the three roles.
struct Plan {
  bool first16;    // first (or only) S MMA is 16-bit
  bool two_phase;  // an 8-bit S is followed by a possible 16-bit S in the same columns
  bool live[2];    // routing half h has a visible pair in this key tile
  bool b16[2];     // bitmask: routing half h is 16-bit
};

// Rows of one sequence: its lengths and where its rows sit in the Q / K / V / O tensors.
struct SeqRows {
  int Lq, Lk;          // this sequence's query and key counts
  int q_row0, k_row0;  // first row in the head plane (0 for dense batches)
  int q_plane, kv_plane;  // head plane of Q / O / lse and of K / V (TMA coordinate 2)
};

// Sequence b, query head h, KV head kvh.  Offsets of a variable-length batch are clipped to
// the tensors, so a malformed offset array cannot move a load or a store out of bounds.
__device__ __forceinline__ SeqRows seq_rows(const AttnParams& p, int b, int h, int kvh) {
  SeqRows s;
  if (p.cu_q) {
    const int q0 = min(max(__ldg(p.cu_q + b), 0), p.q_rows);
    const int k0 = min(max(__ldg(p.cu_k + b), 0), p.k_rows);
    s.Lq = min(max(__ldg(p.cu_q + b + 1) - q0, 0), min(p.Lq, p.q_rows - q0));
    s.Lk = min(max(__ldg(p.cu_k + b + 1) - k0, 0), min(p.Lk, p.k_rows - k0));
    s.q_row0 = q0;
    s.k_row0 = k0;
    s.q_plane = h;
    s.kv_plane = kvh;
  } else {
    s.Lq = p.Lq;
    s.Lk = p.Lk;
    s.q_row0 = s.k_row0 = 0;
    s.q_plane = b * p.H + h;
    s.kv_plane = b * p.Hkv + kvh;
  }
  return s;
}

struct Geo {
  int b, h, kvh, ct, q0, kt_lo, n;
  int half_lo[2], half_hi[2];  // visible key range (union) of each routing half; lo > hi = none
  SeqRows s;
};

// Keys visible to query row i of a sequence of Lq queries and Lk keys: bottom-right causal
// alignment and the sliding window of the kernel arguments.
__device__ __forceinline__ void visible_range(const AttnParams& p, int Lq, int Lk, int i,
                                              int& lo, int& hi) {
  if (!p.causal) {
    lo = 0;
    hi = Lk - 1;
    return;
  }
  const int off = Lk - Lq;
  hi = min(i + off, Lk - 1);
  lo = (p.window > 0) ? max(0, i + off - p.window + 1) : 0;
}

// CTA order: the KV planes are taken in chunks of p.chunk_kv, so that the K / V tiles of the
// CTAs in flight stay resident in L2 while Q and O stream through it; within a chunk, the
// longest query tiles go first (causal), all query heads of the chunk's KV planes side by side.
template <class C>
__device__ __forceinline__ Geo make_geo(const AttnParams& p) {
  Geo g;
  const int G = p.H / p.Hkv;
  const int per_ct = p.chunk_kv * G;         // CTAs of one chunk at one query tile
  const int per_chunk = per_ct * p.n_ct;
  const int idx = blockIdx.x;
  const int chunk = idx / per_chunk;
  int rem = idx - chunk * per_chunk;
  const int ctr = rem / per_ct;
  rem -= ctr * per_ct;
  g.ct = p.n_ct - 1 - ctr;                   // longest-first for causal workloads
  const int kvp = chunk * p.chunk_kv + rem / G;  // KV plane b * Hkv + kvh
  g.b = kvp / p.Hkv;
  g.kvh = kvp - g.b * p.Hkv;
  g.h = g.kvh * G + (rem - (rem / G) * G);
  g.q0 = g.ct * C::MT;
  g.s = seq_rows(p, g.b, g.h, g.kvh);
  const int nh = C::STACK ? 2 : 1;
  int lo_all = 1 << 30, hi_all = -1;
  for (int hh = 0; hh < 2; ++hh) {
    g.half_lo[hh] = 1;
    g.half_hi[hh] = 0;
    if (hh >= nh) continue;
    const int r0 = g.q0 + hh * C::BM;
    const int r1 = min(g.s.Lq, r0 + (C::STACK ? C::BM : C::MT)) - 1;
    if (r0 > r1) continue;
    int lo0, hi0, lo1, hi1;
    visible_range(p, g.s.Lq, g.s.Lk, r0, lo0, hi0);
    visible_range(p, g.s.Lq, g.s.Lk, r1, lo1, hi1);
    const int lo = lo0, hi = hi1;
    if (hi < 0 || lo > hi) continue;
    g.half_lo[hh] = lo;
    g.half_hi[hh] = hi;
    lo_all = min(lo_all, lo);
    hi_all = max(hi_all, hi);
  }
  if (hi_all < lo_all) {
    g.kt_lo = 0;
    g.n = 0;
  } else {
    g.kt_lo = lo_all / C::BN;
    g.n = hi_all / C::BN - g.kt_lo + 1;
  }
  return g;
}

// Key tile kt and its mask group g_idx = kt / group_tiles, advanced without a division.
struct KtPos {
  int kt, g_idx, rem;
  __device__ __forceinline__ void init(const AttnParams& p, int kt0) {
    kt = kt0;
    g_idx = kt0 / p.group_tiles;
    rem = kt0 - g_idx * p.group_tiles;
  }
  __device__ __forceinline__ void next(const AttnParams& p) {
    ++kt;
    if (++rem == p.group_tiles) {
      rem = 0;
      ++g_idx;
    }
  }
};

template <class C>
__device__ __forceinline__ Plan make_plan(const AttnParams& p, const Geo& g, const KtPos& pos) {
  Plan pl;
  const int kt = pos.kt;
  const int c0 = kt * C::BN, c1 = min(g.s.Lk, c0 + C::BN) - 1;
  bool need8 = false, need16 = false;
  const int g_idx = pos.g_idx;
  for (int hh = 0; hh < 2; ++hh) {
    pl.live[hh] = g.half_lo[hh] <= g.half_hi[hh] && g.half_lo[hh] <= c1 && g.half_hi[hh] >= c0;
    pl.b16[hh] = false;
    if (!pl.live[hh] || p.adaptive) continue;
    int bit = 1;
    if (p.mask) {
      const int qt = C::STACK ? 2 * g.ct + hh : g.ct;
      const uint64_t w =
          p.mask[(static_cast<size_t>(g.b * p.H + g.h) * p.nqt + qt) * p.mask_words + (g_idx >> 6)];
      bit = static_cast<int>((w >> (g_idx & 63)) & 1ull);
    }
    pl.b16[hh] = (bit == 0);
    if (bit) need8 = true; else need16 = true;
  }
  if (p.adaptive) {
    pl.first16 = false;
    pl.two_phase = true;
  } else {
    pl.two_phase = need8 && need16;
    pl.first16 = !need8;
  }
  return pl;
}

// ------------------------------------------------------------------ producer ----------

template <class C>
__device__ void producer_role(const AttnParams& p, const Geo& g, uint8_t* smem, Bars& bars,
                              const WaitCtx wc) {
  uint8_t* sQ16 = smem + C::OFF_Q16;
  uint8_t* sQ8 = smem + C::OFF_Q8;
  uint8_t* slots = smem + C::OFF_SLOTS;
  const int pq = g.s.q_plane, pkv = g.s.kv_plane;
  const int qrow = g.s.q_row0 + g.q0;

  prefetch_tmap(&p.tm_q16);
  prefetch_tmap(&p.tm_k16);
  prefetch_tmap(C::PV8 ? &p.tm_v8 : &p.tm_v);
  prefetch_tmap(&p.tm_q8);
  prefetch_tmap(&p.tm_k8);

  mbar_arrive_expect_tx(&bars.q_full, C::Q16_BYTES + C::Q8_BYTES);
  for (int c = 0; c < C::C16; ++c)
    tma_load_3d(sQ16 + c * C::MT * 128, &p.tm_q16, &bars.q_full, c * 64, qrow, pq);
  for (int c = 0; c < C::C8; ++c)
    tma_load_3d(sQ8 + c * C::MT * 128, &p.tm_q8, &bars.q_full, c * 128, qrow, pq);

  uint32_t item = 0;
  bool ok = true;
  // kind: 0 = K8, 1 = K16, 2 = V
  auto load = [&](int kind, int kt) -> bool {
    const int slot = static_cast<int>(item % C::NS);
    const uint32_t use = item / C::NS;
    if (use > 0 && !mbar_wait(&bars.empty[slot], (use - 1) & 1u, wc, W_EMPTY)) return false;
    uint8_t* dst = slots + slot * C::SLOT_BYTES;
    const int row = g.s.k_row0 + kt * C::BN;
    if (kind == 0) {
      mbar_arrive_expect_tx(&bars.full[slot], C::BN * C::D);
      for (int c = 0; c < C::C8; ++c)
        tma_load_3d(dst + c * C::BN * 128, &p.tm_k8, &bars.full[slot], c * 128, row, pkv);
    } else if (C::PV8 && kind == 2) {  // V8: D channel rows of the tile's BN key bytes
      mbar_arrive_expect_tx(&bars.full[slot], C::BN * C::D);
      tma_load_3d(dst, &p.tm_v8, &bars.full[slot], row, 0, pkv);
    } else {
      const CUtensorMap* tm = (kind == 1) ? &p.tm_k16 : &p.tm_v;
      mbar_arrive_expect_tx(&bars.full[slot], C::BN * C::D * 2);
      for (int c = 0; c < C::C16; ++c)
        tma_load_3d(dst + c * C::BN * 128, tm, &bars.full[slot], c * 64, row, pkv);
    }
    ++item;
    return true;
  };

  // Order of the loads = order in which the MMA warp consumes them: the first S operand of
  // tile t+1 before V of tile t; the 16-bit K of a two-phase tile right behind its 8-bit K
  // (separate region Z) or, in shared columns, ahead of the next tile's first operand.
  KtPos pos;
  pos.init(p, g.kt_lo);
  Plan cur = make_plan<C>(p, g, pos);
  ok = load(cur.first16 ? 1 : 0, g.kt_lo);
  if (ok && C::SEP16 && cur.two_phase) ok = load(1, g.kt_lo);
  for (int t = 0; ok && t < g.n; ++t) {
    const int kt = g.kt_lo + t;
    Plan nxt;
    if (!C::SEP16 && cur.two_phase && !(ok = load(1, kt))) break;
    if (t + 1 < g.n) {
      pos.next(p);
      nxt = make_plan<C>(p, g, pos);
      if (!(ok = load(nxt.first16 ? 1 : 0, kt + 1))) break;
      if (C::SEP16 && nxt.two_phase && !(ok = load(1, kt + 1))) break;
    }
    if (!(ok = load(2, kt))) break;
    cur = nxt;
  }
  // Drain: every slot's most recent load must have landed before the CTA may exit.
  const WaitCtx drain{0u, 50000u};  // no abort word: in-flight work always completes
  const uint32_t first = item > static_cast<uint32_t>(C::NS) ? item - C::NS : 0;
  for (uint32_t it = first; it < item; ++it)
    mbar_wait(&bars.full[it % C::NS], (it / C::NS) & 1u, drain, W_DRAIN);
  mbar_wait(&bars.q_full, 0, drain, W_DRAIN);
}

// ------------------------------------------------------------------ MMA issuer --------

template <class C, bool BF16, bool E4M3>
__device__ void mma_role(const AttnParams& p, const Geo& g, uint8_t* smem, Bars& bars,
                         uint32_t tbase, const WaitCtx wc) {
  // The whole warp runs this loop (warp-uniform state and descriptors); the elected lane issues
  // the MMAs, commits and the one plain arrival.  Shared-memory descriptors are built once per
  // operand region and advanced by constant offsets (16-byte units).
  const bool leader = elect_one();
  const uint32_t sQ16 = smem_u32(smem + C::OFF_Q16);
  const uint32_t sQ8 = smem_u32(smem + C::OFF_Q8);
  const uint32_t slots = smem_u32(smem + C::OFF_SLOTS);
  constexpr uint32_t f16 = BF16 ? 1u : 0u;
  constexpr uint32_t id_s16 = idesc(1, f16, f16, 0, 0, C::BN, 128);
  constexpr uint32_t id_s8 = E4M3 ? idesc(1, 0, 0, 0, 0, C::BN, 128) : idesc(2, 1, 1, 0, 0, C::BN, 128);
  constexpr uint32_t id_pv = idesc(1, f16, f16, 0, 1, C::D, 128);
  // 16-bit K-major operands: 128-byte rows (64 elements), row chunks of 64 elements MT * 128 or
  // BN * 128 bytes apart; 8-bit operands likewise (64-byte rows with 64-byte swizzle at D = 64)
  const uint64_t d_q16 = sdesc(sQ16, 16, 1024, SWZ_128B);
  const uint64_t d_k16 = sdesc(slots, 16, 1024, SWZ_128B);
  const uint64_t d_q8 = C::Q8_SW64 ? sdesc(sQ8, 16, 512, SWZ_64B) : sdesc(sQ8, 16, 1024, SWZ_128B);
  const uint64_t d_k8 = C::Q8_SW64 ? sdesc(slots, 16, 512, SWZ_64B) : sdesc(slots, 16, 1024, SWZ_128B);
  const uint64_t d_v = sdesc(slots, C::BN * 128, 1024, SWZ_128B);
  const uint64_t d_p8 = sdesc(smem_u32(smem + C::OFF_P8), 16, 1024, SWZ_128B);
  constexpr uint32_t id_pv8 = idesc(1, 0, 0, 0, 0, C::D, 128);  // E4M3 x E4M3, both K-major
  constexpr uint64_t SLOT_D = C::SLOT_BYTES >> 4;

  uint32_t item = 0;
  // phase bits per S buffer (bit b: buffer b) of the vote barriers; the P barrier of buffer b
  // completes at every use, its phase is (t >> 1) & 1 (registers only: no indexed arrays)
  uint32_t cvb = 0;
  bool ok = mbar_wait(&bars.q_full, 0, wc, W_QFULL);
  tc_fence_after();

  auto take = [&](int& slot) -> bool {
    slot = static_cast<int>(item % C::NS);
    const uint32_t use = item / C::NS;
    ++item;
    if (!mbar_wait(&bars.full[slot], use & 1u, wc, W_FULL)) return false;
    tc_fence_after();
    return true;
  };
  // S of tile t into TMEM column col (its S buffer, or Z)
  auto issue_s = [&](uint32_t col, bool sixteen, int slot) {
    const uint32_t dS = tbase + col;
    if (sixteen) {
      const uint64_t kb = d_k16 + slot * SLOT_D;
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::D / 16; ++s) {
          const uint64_t qo = static_cast<uint64_t>((s >> 2) * ((C::MT * 128) >> 4) + (s & 3) * 2);
          const uint64_t ko = static_cast<uint64_t>((s >> 2) * ((C::BN * 128) >> 4) + (s & 3) * 2);
          mma_f16_ss(dS, d_q16 + qo, kb + ko, id_s16, s > 0 ? 1u : 0u);
        }
      }
    } else {
      const uint64_t kb = d_k8 + slot * SLOT_D;
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::D / 32; ++s) {
          uint64_t qo, ko;
          if (C::Q8_SW64) {
            qo = ko = static_cast<uint64_t>(s * 2);
          } else {
            qo = static_cast<uint64_t>((s >> 2) * ((C::MT * 128) >> 4) + (s & 3) * 2);
            ko = static_cast<uint64_t>((s >> 2) * ((C::BN * 128) >> 4) + (s & 3) * 2);
          }
          if (E4M3)
            mma_f8_ss(dS, d_q8 + qo, kb + ko, id_s8, s > 0 ? 1u : 0u);
          else
            mma_i8_ss(dS, d_q8 + qo, kb + ko, id_s8, s > 0 ? 1u : 0u);
        }
      }
    }
  };
  auto commit = [&](uint64_t* bar) {
    if (leader) tc_commit(bar);
  };
  auto buf = [](int t) { return static_cast<uint32_t>((t & 1) * C::BN); };
  // Separate region Z: the 16-bit S of every two-phase tile goes there right behind the tile's
  // first S (in adaptive mode speculatively: the rows use it only if the tile is flagged).  Z is
  // rewritten once every row has finished with its previous contents (z_free).
  uint32_t zuse = 0;
  auto issue_z = [&]() -> bool {
    int slot16;
    if (zuse > 0) {
      if (!mbar_wait(&bars.z_free, (zuse - 1) & 1u, wc, W_ZFREE)) return false;
      tc_fence_after();
    }
    if (!take(slot16)) return false;
    issue_s(C::TMEM_Z, true, slot16);
    commit(&bars.s16_full[0]);
    commit(&bars.empty[slot16]);
    ++zuse;
    return true;
  };

  KtPos pos;
  pos.init(p, g.kt_lo);
  Plan cur = make_plan<C>(p, g, pos);
  int slot = 0;
  if (ok && (ok = take(slot))) {
    issue_s(buf(0), cur.first16, slot);
    commit(&bars.s_full[0]);
    commit(&bars.empty[slot]);
    if (C::SEP16 && cur.two_phase) ok = issue_z();
  }
  for (int t = 0; ok && t < g.n; ++t) {
    const int bsel = t & 1;
    Plan nxt;
    // Shared columns: a two-phase tile's 16-bit S goes ahead of the next tile's first S, so
    // that the rows waiting for it do not wait for that one too.
    if (!C::SEP16 && cur.two_phase) {
      int slot16;
      if (!(ok = take(slot16))) break;
      if (!(ok = mbar_wait(&bars.vote[bsel], (cvb >> bsel) & 1u, wc, W_VOTE))) break;
      cvb ^= 1u << bsel;
      tc_fence_after();
      bool s16;
      if (p.adaptive) {
        const volatile uint32_t* vv = bars.votes[bsel];
        uint32_t any = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) any |= vv[w];
        s16 = (any & 1u) != 0;  // bit 0 of the vote words: recompute
      } else {
        s16 = true;
      }
      if (s16) {
        issue_s(buf(t), true, slot16);
        commit(&bars.s16_full[bsel]);
        commit(&bars.empty[slot16]);
      } else if (leader) {
        mbar_arrive(&bars.empty[slot16]);
      }
    }
    if (t + 1 < g.n) {
      pos.next(p);
      nxt = make_plan<C>(p, g, pos);
      if (!(ok = take(slot))) break;
      issue_s(buf(t + 1), nxt.first16, slot);
      commit(&bars.s_full[(t + 1) & 1]);
      commit(&bars.empty[slot]);
      if (C::SEP16 && nxt.two_phase && !(ok = issue_z())) break;
    }
    if (!(ok = mbar_wait(&bars.p_full[bsel], static_cast<uint32_t>(t >> 1) & 1u, wc, W_PFULL))) break;
    tc_fence_after();
    int slotv;
    if (!(ok = take(slotv))) break;
    if constexpr (C::PV8) {
      // P8 [128 rows][128 key bytes] and V8 [D rows][128 key bytes], both K-major with 128-byte
      // rows: the operand layout of the E4M3 QK^T; K steps of 32 keys
      const uint64_t pb = d_p8 + static_cast<uint64_t>(bsel * (C::P8_BYTES >> 4));
      const uint64_t vb8 = d_k8 + slotv * SLOT_D;
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::BN / 32; ++s)
          mma_f8_ss(tbase + C::TMEM_O, pb + static_cast<uint64_t>(s * 2),
                    vb8 + static_cast<uint64_t>(s * 2), id_pv8, (t > 0 || s > 0) ? 1u : 0u);
      }
    } else {
      const uint64_t vb = d_v + slotv * SLOT_D;
      const uint32_t pt = tbase + static_cast<uint32_t>(bsel * C::BN);
      // P (16-bit pairs): each softmax column half packs its keys into the first half of its
      // own S columns, so keys [BN/2 * h, BN/2 * (h + 1)) sit at columns BN/2 * h + [0, BN/4)
      constexpr int SPH = C::BN / 32;  // K steps of 16 keys per column half
      if (leader) {
#pragma unroll
        for (int s = 0; s < C::BN / 16; ++s)
          mma_f16_ts(tbase + C::TMEM_O, pt + (s / SPH) * (C::BN / 2) + (s % SPH) * 8,
                     vb + static_cast<uint64_t>(s * ((16 * 128) >> 4)), id_pv,
                     (t > 0 || s > 0) ? 1u : 0u);
      }
    }
    commit(&bars.o_done);
    commit(&bars.empty[slotv]);
    cur = nxt;
  }
  // The epilogue waits for every P.V (the softmax skips most per-tile o_done waits, so that
  // barrier's phase count cannot tell it when the last one is done).
  commit(&bars.o_final);
  // Every MMA issued by this thread must complete before the TMEM is released.
  commit(&bars.drain);
  const WaitCtx drain{0u, 50000u};  // no abort word: in-flight work always completes
  mbar_wait(&bars.drain, 0, drain, W_DRAIN);
}

// Bounded wait by a whole warp: true only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx wc,
                                          uint32_t where) {
  const bool ok = mbar_wait(bar, parity, wc, where);
  return __all_sync(0xFFFFFFFFu, ok);
}

// Debug capture: NCOL words of row `row` of routing tile (bh, qt, kt), starting at column col0,
// into the caller's slot for that tile, if it has one (base null: that kind is not captured).
template <int NCOL>
__device__ __forceinline__ void dbg_dump(const AttnParams& p, uint32_t* base, int bm, int bn,
                                         int bh, int qt, int kt, int row, int col0,
                                         const uint32_t* raw) {
  if (base == nullptr || qt >= p.nqt || kt >= p.nkt) return;
  const int s = __ldg(p.dbg_slot + (static_cast<size_t>(bh) * p.nqt + qt) * p.nkt + kt);
  if (s < 0 || s >= p.dbg_nslots) return;
  uint32_t* dst = base + (static_cast<size_t>(s) * bm + row) * bn + col0;
#pragma unroll
  for (int c = 0; c < NCOL; c += 4)
    st_global_v4(dst + c, make_uint4(raw[c], raw[c + 1], raw[c + 2], raw[c + 3]));
}

// (packed f32x2 helpers: ptx.cuh)
// 2^x for a pair on the FMA and ALU pipes instead of the MUFU: 2^x = 2^n * 2^f with n = rint(x)
// (magic-number rounding) and f = x - n in [-1/2, 1/2], 2^f from a degree-3 polynomial fitted
// to it for least relative error on that interval (max 7.7e-5, below the 16-bit rounding of
// P), and n added to the exponent field.  x < -125 gives 0, as the flush-to-zero MUFU ex2 does
// below -126 (masked scores are -inf).
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float& p0, float& p1) {
  auto two = [](float v) { return f2_pack(v, v); };
  const uint64_t M2 = two(12582912.0f);  // 1.5 * 2^23
  const uint64_t xx = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t tt = f2_add(xx, M2);
  const uint64_t fr = f2_sub(xx, f2_sub(tt, M2));
  uint64_t pp = f2_fma(two(0.05518098175525665f), fr, two(0.2426345944404602f));
  pp = f2_fma(pp, fr, two(0.6932613253593445f));
  pp = f2_fma(pp, fr, two(0.9999262094497681f));
  float r0, r1, t0, t1;
  f2_unpack(pp, r0, r1);
  f2_unpack(tt, t0, t1);
  p0 = (x0 < -125.0f) ? 0.0f : __uint_as_float(__float_as_uint(r0) + (__float_as_uint(t0) << 23));
  p1 = (x1 < -125.0f) ? 0.0f : __uint_as_float(__float_as_uint(r1) + (__float_as_uint(t1) << 23));
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// acc + the low / high 16-bit half of a packed pair (bf16 or fp16), one rounding: sums the
// rounded P values as the P.V MMA sees them, without unpacking them.
template <bool BF16>
__device__ __forceinline__ float add_lo16(float acc, uint32_t pk) {
  float r;
  if (BF16) asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.bf16 %0, lo, %2;\n\t}" : "=f"(r) : "r"(pk), "f"(acc));
  else asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, lo, %2;\n\t}" : "=f"(r) : "r"(pk), "f"(acc));
  return r;
}
template <bool BF16>
__device__ __forceinline__ float add_hi16(float acc, uint32_t pk) {
  float r;
  if (BF16) asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.bf16 %0, hi, %2;\n\t}" : "=f"(r) : "r"(pk), "f"(acc));
  else asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tadd.rn.f32.f16 %0, hi, %2;\n\t}" : "=f"(r) : "r"(pk), "f"(acc));
  return r;
}

// Two threads per row of the 128-row MMA tile (the TMEM lane): the thread of column half h
// (warps 4h .. 4h + 3) handles key columns [BN/2 * h, BN/2 * (h + 1)) of each key tile.  Per
// key tile: read its half row of S, turn it into fp32 values of the raw product (exact int32 ->
// fp32 for INT8 tiles; E4M3 and 16-bit tiles accumulate in fp32), mask, take the half-row max
// and combine it with the partner's through shared memory (an mbarrier per lane quadrant, so
// that every wait is bounded; the exchange slots alternate with the S buffer), vote (look-ahead
// rule), exponentiate against a lazy reference max (it moves only when the row max exceeds it
// by more than 8 in log2 units, so O is rarely rescaled), pack P as 16-bit pairs into the first
// half of the thread's own S columns (each 32-column chunk stored when ready), and keep two
// partial row sums: of the exact p (for lse) and of the rounded p that the P.V MMA multiplies
// (for O).  Both threads of a row take identical decisions from identical inputs.
template <class C, bool BF16, bool E4M3, bool SKIP, bool DBG>
__device__ void softmax_role(const AttnParams& p, const Geo& g, uint8_t* smem, Bars& bars,
                             uint32_t tbase, const WaitCtx wc) {
  constexpr int N = C::BN, NH = C::BN / 2;
  // lazy reference max (the O rescale only when a row max passes it by 8); the 8-bit P.V mode
  // takes its exponentials against the exact running max (the rounding of p to E4M3 is defined
  // against it)
  constexpr float RESCALE_THRESH = C::PV8 ? 0.0f : 8.0f;
  // At D = 128 the two partner warps of a row run their exponentials in lock step on one SM
  // sub-partition's MUFU; moving one pair in eight to the FMA pipe shortens that phase (at
  // D = 256 the tensor core sets the pace and the extra instructions cost more than they save).
  constexpr bool POLY_EX2 = (C::D == 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = warp >> 2;   // column half
  const int q4 = warp & 3;   // TMEM lane quadrant
  const int r = q4 * 32 + lane;
  const int i = g.q0 + r;
  const bool row_valid = i < g.s.Lq;
  const int hh = C::STACK ? (r >> 6) : 0;
  const int qt_r = C::STACK ? 2 * g.ct + hh : g.ct;
  const int bh_q = g.b * p.H + g.h;
  const uint32_t lane_base = tbase + (static_cast<uint32_t>(q4 * 32) << 16);
  int lo_r = 1, hi_r = 0;
  if (row_valid) visible_range(p, g.s.Lq, g.s.Lk, i, lo_r, hi_r);
  const float sq = (row_valid && qt_r < p.nqt) ? __ldg(p.q_scale + static_cast<size_t>(bh_q) * p.nqt + qt_r) : 0.0f;
  const float* ks_row = p.k_scale + static_cast<size_t>(g.b * p.Hkv + g.kvh) * p.nkt;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float sq_scale = sq * p.scale_log2;
  const uint32_t xch = smem_u32(smem + C::OFF_XCH) + static_cast<uint32_t>(r * 4);
  uint64_t* xbar = &bars.xbar[q4];

  float m_ref = NEG_INF;   // max used for the exponentials (lazy)
  float m_true = NEG_INF;  // true running max of the used scores (look-ahead rule)
  float l_ex = 0.0f, l_rd = 0.0f;
  // phase bits per S buffer (bit b: buffer b) of the vote and 16-bit S barriers; the S barrier
  // of buffer b completes at every use, its phase is (t >> 1) & 1
  uint32_t cvb = 0, c16b = 0, nx = 0;
  uint32_t zc = 0;  // uses of the separate 16-bit region Z so far
  bool ok = true;
  uint32_t raw[NH];
  // debug capture of this thread's half row of a live routing tile's raw S (capture build only)
  const int row_in_tile = C::STACK ? (r & 63) : r;
  auto dump = [&](bool s16, bool live, int kt) {
    if constexpr (DBG) {
      if (live)
        dbg_dump<NH>(p, s16 ? p.dbg_s16 : p.dbg_s8, C::BM, N, bh_q, qt_r, kt, row_in_tile,
                     h * NH, raw);
    }
  };

  // Publish v in this thread's exchange slot of parity `par` and return the partner's value.
  // The slot's previous value (two key tiles back) has been read: the partner read it before
  // it published that tile's P, which the MMA warp waited for before issuing this tile's S.
  auto exchange = [&](int par, float v, float& other) -> bool {
    sts_u32(xch + static_cast<uint32_t>((par * 2 + h) * C::MT * 4), __float_as_uint(v));
    mbar_arrive(xbar);
    if (!mbar_wait(xbar, nx & 1u, wc, W_XCH)) return false;
    ++nx;
    other = __uint_as_float(lds_u32(xch + static_cast<uint32_t>((par * 2 + (h ^ 1)) * C::MT * 4)));
    return true;
  };
  auto load_s = [&](int col) {  // this thread's half row of the S at TMEM column col
#pragma unroll
    for (int c = 0; c < NH / 32; ++c)
      tmem_ld32(lane_base + static_cast<uint32_t>(col + h * NH + c * 32),
                *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
    tmem_wait_ld();
  };
  auto int_to_float = [&]() {  // exact: |int32 product| < 2^22
#pragma unroll
    for (int c = 0; c < NH; ++c) raw[c] = __float_as_uint(static_cast<float>(static_cast<int>(raw[c])));
  };
  auto apply_mask = [&](int j0) {  // keep the row's visible columns of this half, -inf elsewhere
    const int a = row_valid ? lo_r - j0 : NH;
    const int b = row_valid ? hi_r - j0 : -1;
#pragma unroll
    for (int c = 0; c < NH; ++c) raw[c] = (c < a || c > b) ? 0xff800000u : raw[c];
  };
  auto raw_max = [&]() -> float {
    float m0 = NEG_INF, m1 = NEG_INF;
#pragma unroll
    for (int c = 0; c < NH; c += 4) {
      m0 = max3(m0, __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
      m1 = max3(m1, __uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3]));
    }
    return fmaxf(m0, m1);
  };

  auto load_s_async = [&](int col) {  // as load_s, without the wait for the data
#pragma unroll
    for (int c = 0; c < NH / 32; ++c)
      tmem_ld32(lane_base + static_cast<uint32_t>(col + h * NH + c * 32),
                *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
  };
  // the key block's scale is read one tile ahead (its L2 latency would otherwise sit on the
  // path of every tile)
  float ks_nxt = (g.n > 0) ? __ldg(ks_row + g.kt_lo) : 0.0f;
  // the routing plan is likewise made one tile ahead (its mask read and arithmetic then overlap
  // the current tile's work)
  KtPos pos;
  pos.init(p, g.kt_lo);
  Plan pl_nxt = make_plan<C>(p, g, pos);

  for (int t = 0; ok && t < g.n; ++t) {
    const int kt = g.kt_lo + t;
    const int bsel = t & 1;
    const Plan pl = pl_nxt;
    const float ks_cur = ks_nxt;
    if (t + 1 < g.n) {
      ks_nxt = __ldg(ks_row + kt + 1);
      pos.next(p);
      pl_nxt = make_plan<C>(p, g, pos);
    }
    if (!(ok = warp_wait(&bars.s_full[bsel], static_cast<uint32_t>(t >> 1) & 1u, wc, W_SFULL))) break;
    tc_fence_after();
    const int j0 = kt * N + h * NH;
    const bool full = row_valid && j0 >= lo_r && j0 + NH - 1 <= hi_r;
    // (a zero block scale would turn masked -inf entries into NaN: keep it positive)
    const float cs8 = fmaxf(sq_scale * ks_cur, 1e-30f);
    bool sixteen = pl.first16, my16 = pl.first16;
    bool drop = false;  // this row's routing tile is dropped by the threshold skip
    float cscale, tmax, other;
    if (C::SEP16 && pl.two_phase) {
      // The 16-bit S is in Z, issued with the tile.  Look-ahead mode: vote on the 8-bit half-row
      // maximum (a row reaches m - tau iff one of its halves does, so the tile vote needs no
      // exchange), read Z while the vote completes, and fall back to the 8-bit S only if the
      // tile is not flagged.  Mixed stacked halves know their precision from the mask.
      const bool live_mine = hh ? pl.live[1] : pl.live[0];
      if (p.adaptive) {
        load_s(bsel * N);
        dump(false, live_mine, kt);
        if (!E4M3) int_to_float();
        if (!full) apply_mask(j0);
        const float hmax = raw_max();
        const float t8 = (hmax == NEG_INF) ? NEG_INF : hmax * cs8;
        // vote word: bit 0 recompute (some row within tau of its running max), bit 1 keep (some
        // row within skip_tau, or without a running max yet); a routing tile whose rows all
        // miss bit 1 is dropped
        const bool vote = (t8 != NEG_INF) && (t8 >= m_true - p.tau_log2);
        uint32_t wv = __any_sync(0xFFFFFFFFu, vote) ? 1u : 0u;
        if (SKIP) {
          const bool keep = (t8 != NEG_INF) && (m_true == NEG_INF || t8 >= m_true - p.skip_log2);
          wv |= __any_sync(0xFFFFFFFFu, keep) ? 2u : 0u;
        }
        if (lane == 0) bars.votes[bsel][warp] = wv;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.vote[bsel]);
        if (!(ok = warp_wait(&bars.s16_full[0], zc & 1u, wc, W_S16))) break;
        tc_fence_after();
        load_s_async(C::TMEM_Z);
        ok = warp_wait(&bars.vote[bsel], (cvb >> bsel) & 1u, wc, W_VOTE);
        tmem_wait_ld();
        if (!ok) break;
        cvb ^= 1u << bsel;
        const volatile uint32_t* vv = bars.votes[bsel];
        uint32_t v0, v1;
        if (C::STACK) {  // rows 0-63: quadrants 0, 1; rows 64-127: quadrants 2, 3
          v0 = vv[0] | vv[1] | vv[4] | vv[5];
          v1 = vv[2] | vv[3] | vv[6] | vv[7];
        } else {
          v0 = v1 = vv[0] | vv[1] | vv[2] | vv[3] | vv[4] | vv[5] | vv[6] | vv[7];
        }
        const uint32_t vw = hh ? v1 : v0;
        drop = SKIP && (vw & 2u) == 0;
        my16 = (vw & 1u) != 0 && !drop;
        if (my16) dump(true, live_mine, kt);  // raw holds the 16-bit S of region Z
        if (!my16 && !drop) {  // not flagged: back to the 8-bit scores (still in this tile's S buffer)
          load_s(bsel * N);
          if (!E4M3) int_to_float();
        }
      } else {
        my16 = hh ? (pl.live[1] && pl.b16[1]) : (pl.live[0] && pl.b16[0]);
        if (my16) {
          if (!(ok = warp_wait(&bars.s16_full[0], zc & 1u, wc, W_S16))) break;
          tc_fence_after();
          load_s(C::TMEM_Z);
          dump(true, live_mine, kt);
        } else {
          load_s(bsel * N);
          dump(false, live_mine, kt);
          if (!E4M3) int_to_float();
        }
      }
      // (a warp that skipped the s16_full wait cannot fall two phases behind: the next use of
      // Z needs its z_free arrival)
      ++zc;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.z_free);
      sixteen = my16;
      cscale = my16 ? p.scale_log2 : cs8;
      tmax = NEG_INF;
      if (!drop) {  // (both threads of a row take the same branch)
        if (!full) apply_mask(j0);
        tmax = raw_max();
        if (!(ok = exchange(bsel, tmax, other))) break;
        tmax = fmaxf(tmax, other);
      }
    } else {
      load_s(bsel * N);
      // (a two-phase tile here reads its 8-bit S first; in bitmask mode that S belongs to the
      // 8-bit routing half only)
      dump(sixteen, (hh ? pl.live[1] : pl.live[0]) &&
                        (sixteen || p.adaptive || !(hh ? pl.b16[1] : pl.b16[0])), kt);
      cscale = sixteen ? p.scale_log2 : cs8;
      if (!sixteen && !E4M3) int_to_float();
      if (!full) apply_mask(j0);
      tmax = raw_max();
      if (!(ok = exchange(bsel, tmax, other))) break;
      tmax = fmaxf(tmax, other);
    }
    if (!C::SEP16 && pl.two_phase) {
      if (p.adaptive) {  // vote word as above: bit 0 recompute, bit 1 keep
        const float t8 = (tmax == NEG_INF) ? NEG_INF : tmax * cscale;
        const bool vote = (t8 != NEG_INF) && (t8 >= m_true - p.tau_log2);
        uint32_t wv = __any_sync(0xFFFFFFFFu, vote) ? 1u : 0u;
        if (SKIP) {
          const bool keep = (t8 != NEG_INF) && (m_true == NEG_INF || t8 >= m_true - p.skip_log2);
          wv |= __any_sync(0xFFFFFFFFu, keep) ? 2u : 0u;
        }
        if (lane == 0) bars.votes[bsel][warp] = wv;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.vote[bsel]);
      if (!(ok = warp_wait(&bars.vote[bsel], (cvb >> bsel) & 1u, wc, W_VOTE))) break;
      cvb ^= 1u << bsel;
      bool f0, f1;
      if (p.adaptive) {
        const volatile uint32_t* vv = bars.votes[bsel];
        uint32_t v0, v1;
        if (C::STACK) {  // rows 0-63: quadrants 0, 1; rows 64-127: quadrants 2, 3
          v0 = vv[0] | vv[1] | vv[4] | vv[5];
          v1 = vv[2] | vv[3] | vv[6] | vv[7];
        } else {
          v0 = v1 = vv[0] | vv[1] | vv[2] | vv[3] | vv[4] | vv[5] | vv[6] | vv[7];
        }
        f0 = (v0 & 1u) != 0;
        f1 = (v1 & 1u) != 0;
        drop = SKIP && ((hh ? v1 : v0) & 2u) == 0;
      } else {
        f0 = pl.live[0] && pl.b16[0];
        f1 = pl.live[1] && pl.b16[1];
      }
      const bool s16 = p.adaptive ? (f0 || f1) : true;
      my16 = (hh ? f1 : f0) && !drop;
      if (s16) {
        if (!(ok = warp_wait(&bars.s16_full[bsel], (c16b >> bsel) & 1u, wc, W_S16))) break;
        c16b ^= 1u << bsel;
        tc_fence_after();
        if (my16) {  // (both threads of a row take this branch or neither)
          load_s(bsel * N);
          dump(true, hh ? pl.live[1] : pl.live[0], kt);
          sixteen = true;
          cscale = p.scale_log2;
          if (!full) apply_mask(j0);
          tmax = raw_max();
          if (!(ok = exchange(bsel, tmax, other))) break;
          tmax = fmaxf(tmax, other);
        }
      }
    }
    if (p.route && h == 0 && lane == 0 && (q4 == 0 || (C::STACK && q4 == 2))) {
      if (hh ? pl.live[1] : pl.live[0]) {
        const uint8_t v = drop ? 4 : my16 ? (pl.two_phase && p.adaptive ? 3 : 2) : 1;
        p.route[(static_cast<size_t>(bh_q) * p.nqt + qt_r) * p.nkt + kt] = v;
      }
    }

    const float tl = (drop || tmax == NEG_INF) ? NEG_INF : tmax * cscale;  // log2 units
    m_true = fmaxf(m_true, tl);
    const bool move = (tl != NEG_INF) && (m_ref == NEG_INF || tl > m_ref + RESCALE_THRESH);
    const float new_ref = move ? tl : m_ref;
    const float alpha = move ? ((m_ref == NEG_INF) ? 0.0f : ex2(m_ref - new_ref)) : 1.0f;
    l_ex *= alpha;
    l_rd *= alpha;
    m_ref = new_ref;

    // p = 2^(value * cscale - m_ref); masked entries hold -inf and give 0.  Each 32-column
    // chunk of P (16 packed columns) goes into this tile's S buffer as soon as it is ready: P.V
    // of the tile two steps back, which read that buffer, completed before S was written.
    if constexpr (C::PV8) {
      // 8-bit P: p * 2^8 rounded to E4M3 (the running max's own p is 256 < 448), into this
      // tile's P8 buffer, row r, keys [NH * h, NH * h + NH) = 16-byte units 4h .. 4h + 3,
      // XOR-swizzled by r & 7 (the 128-byte swizzle of a K-major operand).  P.V of the tile two
      // steps back, which read this buffer, completed before S(t) was written.
      const uint32_t prow = smem_u32(smem + C::OFF_P8) + static_cast<uint32_t>(bsel * C::P8_BYTES) +
                            static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128);
      const float mu = (m_ref == NEG_INF) ? 0.0f : m_ref;
      const uint64_t c2 = f2_pack(cscale, cscale);
      const uint64_t nb2 = f2_pack(-mu, -mu);
      uint64_t se0 = 0, se1 = 0;
      float sr0 = 0.f, sr1 = 0.f, sr2 = 0.f, sr3 = 0.f;
      uint32_t w[4];
#pragma unroll
      for (int c = 0; c < NH; c += 4) {
        float x0, x1, x2, x3, p0, p1, p2, p3;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), c2, nb2),
                  x0, x1);
        f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3])), c2, nb2),
                  x2, x3);
        p0 = drop ? 0.0f : ex2(x0);
        p1 = drop ? 0.0f : ex2(x1);
        p2 = drop ? 0.0f : ex2(x2);
        p3 = drop ? 0.0f : ex2(x3);
        se0 = f2_add(se0, f2_pack(p0, p1));
        se1 = f2_add(se1, f2_pack(p2, p3));
        const uint32_t lo = e4m3x2(p0 * 256.0f, p1 * 256.0f), hi = e4m3x2(p2 * 256.0f, p3 * 256.0f);
        const uint32_t flo = e4m3x2_to_f16x2(lo), fhi = e4m3x2_to_f16x2(hi);
        sr0 = add_lo16<false>(sr0, flo);
        sr1 = add_hi16<false>(sr1, flo);
        sr2 = add_lo16<false>(sr2, fhi);
        sr3 = add_hi16<false>(sr3, fhi);
        w[(c >> 2) & 3] = lo | (hi << 16);
        if ((c & 15) == 12) {
          const uint32_t u = static_cast<uint32_t>(4 * h + (c >> 4));
          st_shared_v4(prow + ((u ^ static_cast<uint32_t>(r & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
      }
      if (!drop) {
        float a0, a1;
        f2_unpack(f2_add(se0, se1), a0, a1);
        l_ex += a0 + a1;
        // the rounded p carry the factor 2^8; O is divided by this sum, so it cancels
        l_rd += (sr0 + sr1) + (sr2 + sr3);
      }
      fence_proxy_async_smem();  // the P.V MMA reads P8 through the async proxy
    } else if (drop) {  // a dropped routing tile: P = 0 for this row, (m, l) unchanged
      const uint32_t zero[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < NH / 32; ++c)
        tmem_st16(lane_base + static_cast<uint32_t>(bsel * N + h * NH + c * 16), zero);
    } else {
      const float mu = (m_ref == NEG_INF) ? 0.0f : m_ref;
      const uint64_t c2 = f2_pack(cscale, cscale);
      const uint64_t nb2 = f2_pack(-mu, -mu);
      uint64_t se0 = 0, se1 = 0;
      float sr0 = 0.f, sr1 = 0.f, sr2 = 0.f, sr3 = 0.f;
#pragma unroll
      for (int c = 0; c < NH; c += 2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), c2, nb2),
                  x0, x1);
        float p0, p1;
        if (POLY_EX2 && ((c >> 1) & 7) == 7) {  // one pair in eight on the FMA pipe
          ex2_poly2(x0, x1, p0, p1);
        } else {
          p0 = ex2(x0);
          p1 = ex2(x1);
        }
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
        if ((c & 31) == 30)
          tmem_st16(lane_base + static_cast<uint32_t>(bsel * N + h * NH + (c >> 5) * 16),
                    &raw[(c >> 5) * 16]);
      }
      {
        float a0, a1;
        f2_unpack(f2_add(se0, se1), a0, a1);
        l_ex += a0 + a1;
        l_rd += (sr0 + sr1) + (sr2 + sr3);
      }
    }

    // O is rescaled (rarely: lazy reference max) once P.V of the previous tile has completed.
    // The wait is exact although most tiles skip it: S(t), seen complete above, was issued
    // after P.V(t-2) and the tensor core completes in issue order, and P.V(t) is issued only
    // after this warp's P arrival below, so o_done stands at phase t-1 or t.
    if (t > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
      if (!(ok = warp_wait(&bars.o_done, (t - 1) & 1u, wc, W_ODONE))) break;
      tc_fence_after();
      {  // each thread rescales its half of O
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t ov[16];
          const uint32_t ta = lane_base + static_cast<uint32_t>(C::TMEM_O + h * (C::D / 2) + c * 16);
          tmem_ld16(ta, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float lo, hi;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(ov[e]), __uint_as_float(ov[e + 1])), a2, 0ull),
                      lo, hi);
            ov[e] = __float_as_uint(lo);
            ov[e + 1] = __float_as_uint(hi);
          }
          tmem_st16(ta, ov);
        }
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.p_full[bsel]);
  }
  if (!ok) return;

  // epilogue: combine the two halves' row sums, then O / l and lse
  if (g.n > 0) {
    if (!warp_wait(&bars.o_final, 0, wc, W_ODONE)) return;
    tc_fence_after();
  }
  const int par = g.n & 1;  // the exchange slots of parity n & 1 were last read two tiles back
  float other_rd, other_ex;
  if (!exchange(par, l_rd, other_rd)) return;
  mbar_arrive(xbar);  // a phase without a write: both partners have read the l_rd slots
  if (!mbar_wait(xbar, nx & 1u, wc, W_XCH)) return;
  ++nx;
  if (!exchange(par, l_ex, other_ex)) return;
  const float l_rd_t = l_rd + other_rd, l_ex_t = l_ex + other_ex;
  const float inv = (l_rd_t > 0.0f) ? 1.0f / l_rd_t : 0.0f;
  constexpr int DH = C::D / 2;
  const size_t orow =
      (static_cast<size_t>(g.s.q_plane) * p.q_rows + g.s.q_row0 + (row_valid ? i : 0)) * C::D + h * DH;
  // At D = 256 (128 KB of O per tile) O leaves through shared memory; at D <= 128 each thread
  // stores its own row (measured: staging gains 4% at D = 256 and nothing at D = 128).
  constexpr bool STAGE_O = C::D == 256;
  if (STAGE_O && g.n > 0) {
    // O leaves through shared memory so that every warp store writes whole 128-byte lines (a
    // thread's own row lies one row pitch away from its neighbours').  Every operand in shared
    // memory has been consumed (o_final), so Q and the ring hold the staging area: row r of
    // the tile at r * RB bytes, its 16-byte units XOR-swizzled by r & 7, so that 32 rows
    // writing the same unit and one warp reading 32 consecutive units hit distinct banks.
    const uint32_t es = p.out_f32 ? 4u : 2u, RB = C::D * es;
    const uint32_t stg = smem_u32(smem), rbase = stg + static_cast<uint32_t>(r) * RB;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll 1
    for (int c = 0; c < DH / 32; ++c) {
      uint32_t ov[32];
      tmem_ld32(lane_base + static_cast<uint32_t>(C::TMEM_O + h * DH + c * 32), ov);
      tmem_wait_ld();
      auto sc = [&](int e) { return __float_as_uint(__uint_as_float(ov[e]) * inv); };
      if (p.out_f32) {
        const uint32_t u0 = static_cast<uint32_t>(h * DH + c * 32) / 4;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_shared_v4(rbase + (((u0 + k) ^ sw) << 4), sc(4 * k), sc(4 * k + 1), sc(4 * k + 2),
                       sc(4 * k + 3));
      } else {
        const uint32_t u0 = static_cast<uint32_t>(h * DH + c * 32) / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(ov[8 * k + 2 * q]) * inv;
            const float b2 = __uint_as_float(ov[8 * k + 2 * q + 1]) * inv;
            if (BF16) {
              __nv_bfloat162 v2 = __floats2bfloat162_rn(a, b2);
              w[q] = *reinterpret_cast<uint32_t*>(&v2);
            } else {
              __half2 v2 = __floats2half2_rn(a, b2);
              w[q] = *reinterpret_cast<uint32_t*>(&v2);
            }
          }
          st_shared_v4(rbase + (((u0 + k) ^ sw) << 4), w[0], w[1], w[2], w[3]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.ostage);
    if (!warp_wait(&bars.ostage, 0, wc, W_OSTAGE)) return;
    // the eight softmax warps (threads 0-255) copy the tile out, 16 bytes per thread, rows past
    // the sequence skipped
    const int UPR = static_cast<int>(RB / 16);
    const size_t row0 = static_cast<size_t>(g.s.q_plane) * p.q_rows + g.s.q_row0 + g.q0;
    uint8_t* obase = static_cast<uint8_t*>(p.o);
    for (int L = static_cast<int>(threadIdx.x); L < C::MT * UPR; L += 256) {
      const int row = L / UPR, u = L - row * UPR;
      const uint4 v = ld_shared_v4(stg + static_cast<uint32_t>(row) * RB +
                                   ((static_cast<uint32_t>(u) ^ static_cast<uint32_t>(row & 7)) << 4));
      if (g.q0 + row < g.s.Lq)
        st_global_v4(obase + (row0 + row) * C::D * es + static_cast<size_t>(u) * 16, v);
    }
  } else {
    // 8-bit P.V: O carries V's per-channel scale, applied here
    const float* svp = C::PV8 ? p.v_scale + static_cast<size_t>(g.s.kv_plane) * C::D + h * DH : nullptr;
#pragma unroll 1
    for (int c = 0; c < DH / 32; ++c) {
      uint32_t ov[32];
      if (g.n > 0) {
        tmem_ld32(lane_base + static_cast<uint32_t>(C::TMEM_O + h * DH + c * 32), ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = 0u;
      }
      if (!row_valid) continue;
      if constexpr (C::PV8) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          ov[e] = __float_as_uint(__uint_as_float(ov[e]) * __ldg(svp + c * 32 + e));
      }
      // 32-byte stores: each thread writes whole sectors of its row
      auto sc = [&](int e) { return __float_as_uint(__uint_as_float(ov[e]) * inv); };
      if (p.out_f32) {
        float* dst = static_cast<float*>(p.o) + orow + c * 32;
#pragma unroll
        for (int e = 0; e < 32; e += 8)
          st_global_v8(dst + e, sc(e), sc(e + 1), sc(e + 2), sc(e + 3), sc(e + 4), sc(e + 5), sc(e + 6),
                       sc(e + 7));
      } else {
        uint16_t* dst = static_cast<uint16_t*>(p.o) + orow + c * 32;
#pragma unroll
        for (int e = 0; e < 32; e += 16) {
          uint32_t w[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float a = __uint_as_float(ov[e + 2 * q]) * inv;
            const float b2 = __uint_as_float(ov[e + 2 * q + 1]) * inv;
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
  }
  if (h == 0 && row_valid && p.lse) {
    p.lse[static_cast<size_t>(g.s.q_plane) * p.q_rows + g.s.q_row0 + i] =
        (l_ex_t > 0.0f) ? m_ref * 0.69314718055994530942f + logf(l_ex_t) : NEG_INF;
  }
}

// ------------------------------------------------------------------ kernel ------------

template <class C, bool BF16, bool E4M3, bool SKIP, bool DBG>
__global__ void __launch_bounds__(C::THREADS, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the layouts need a 1024-aligned base
    if (threadIdx.x == 0) atomicOr(&g_lamp_error, 0x4u);
    return;
  }
  Bars& bars = *reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5;
  const Geo g = make_geo<C>(p);

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.s_full[b], 1);
      mbar_init(&bars.s16_full[b], 1);
      mbar_init(&bars.vote[b], 8);
      mbar_init(&bars.p_full[b], 8);
    }
    mbar_init(&bars.o_done, 1);
    mbar_init(&bars.drain, 1);
    mbar_init(&bars.z_free, 8);
    mbar_init(&bars.o_final, 1);
    mbar_init(&bars.ostage, 8);
    for (int q = 0; q < 4; ++q) mbar_init(&bars.xbar[q], 64);
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

  if (warp == 8) {
    if ((threadIdx.x & 31) == 0 && g.n > 0) producer_role<C>(p, g, smem, bars, wc);
  } else if (warp == 9) {
    if (g.n > 0) mma_role<C, BF16, E4M3>(p, g, smem, bars, tbase, wc);
  } else {
    softmax_role<C, BF16, E4M3, SKIP, DBG>(p, g, smem, bars, tbase, wc);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) {
    __syncwarp();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

// A one-block kernel whose single wait can never complete: exercises the bounded-wait error
// path (records a timeout in the error word and returns) without faulting the GPU.
__global__ void selftest_timeout_kernel(uint64_t wait_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx w{smem_u32(&abort_flag), static_cast<uint32_t>(wait_ns / 1000)};
    mbar_wait(&bar, 0, w, W_SELFTEST);
  }
  __syncthreads();
}

// Evaluates the kernels' exponentials on a list of inputs (so that they can be checked against
// the mathematical 2^x): method 0 = ex2_poly2 (the FMA-pipe polynomial), 1 = ex2 (MUFU).
__global__ void exp2_eval_kernel(const float* x, float* y, int n, int method) {
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * gridDim.x * blockDim.x) {
    const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : x[i];
    float p0, p1;
    if (method == 0) {
      ex2_poly2(x0, x1, p0, p1);
    } else {
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    y[i] = p0;
    if (i + 1 < n) y[i + 1] = p1;
  }
}

}  // namespace lamp
