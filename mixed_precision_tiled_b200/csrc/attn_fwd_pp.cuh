// Routed mixed-precision attention forward, head dimension 128, INT8 8-bit format: two query
// tiles per CTA.  (FP8 E4M3 runs in the single-tile kernel of attn_fwd.cuh.)
//
// Same computation as attn_fwd.cuh (TileMix page, section 2 "How It Works": 8-bit or 16-bit
// score tiles chosen per tile, one shared online softmax; LampAttention abstract: 8-bit
// products, look-ahead recomputation of sensitive tiles in 16 bits), organised for B200 so
// that the tensor core works on one query tile while the softmax works on the other:
//   * a CTA owns two 128-row query tiles A and B of one (batch, head) and streams each key
//     tile (K8 and/or K16, V) through shared memory once for both;
//   * TMEM holds S_A, S_B (128 columns each) and O_A, O_B (128 each) = all 512 columns;
//   * warpgroup 0 runs the softmax of A, warpgroup 1 that of B (one row per thread); warp 8
//     issues TMA loads, warp 9 issues the MMAs in the order
//       S_A(0) S_B(0) | PV_A(t) S_A(t+1) PV_B(t) S_B(t+1) | ...
//     so that while one warpgroup exponentiates tile t, the tensor core runs the other tile's
//     P.V and next QK^T;
//   * softmax arithmetic: row max over raw int32 accumulators (integer max), exact
//     int->float conversion by the 2^23 magic-number add (ALU + FMA pipes instead of the
//     MUFU conversion), packed f32x2 FMAs / adds, tree reductions, and a lazy O rescale: the
//     reference max used for the exponentials only moves when a row max exceeds it by more
//     than 8 (log2 units), which keeps P <= 256 and makes the TMEM round trip of O rare; the
//     true running max is tracked separately for the look-ahead rule.
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
  static constexpr int SLOT_BYTES = BN * D * 2;
  static constexpr int NS = 4;
  static constexpr int OFF_Q16 = 0;                      // + X * Q16_BYTES
  static constexpr int OFF_Q8 = 2 * Q16_BYTES;           // + X * Q8_BYTES
  static constexpr int OFF_SLOTS = 2 * (Q16_BYTES + Q8_BYTES);
  static constexpr int OFF_BAR = OFF_SLOTS + NS * SLOT_BYTES;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
  static constexpr int TMEM_COLS = 512;
  static constexpr float RESCALE_THRESH = 8.0f;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(OFF_SLOTS % 1024 == 0 && OFF_Q8 % 1024 == 0, "alignment");
};

struct PPBars {
  uint64_t q_full;
  uint64_t full[PPCfg::NS];
  uint64_t empty[PPCfg::NS];
  uint64_t s_full[2];
  uint64_t s16_full[2];
  uint64_t vote[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort;
  uint32_t votes[2][4];
};

struct PPGeo {
  int b, h, kvh, pair, q0, kt_lo, n;
  int lo[2], hi[2];  // visible key range (union) of query tile X; lo > hi = none
};

__device__ __forceinline__ PPGeo pp_geo(const AttnParams& p) {
  PPGeo g;
  const int BH = p.B * p.H;
  const int idx = blockIdx.x;
  const int n_pairs = (p.nqt + 1) / 2;
  g.pair = n_pairs - 1 - idx / BH;  // longest-first
  const int bh = idx - (idx / BH) * BH;
  g.b = bh / p.H;
  g.h = bh - g.b * p.H;
  g.kvh = g.h / (p.H / p.Hkv);
  g.q0 = g.pair * 2 * PPCfg::MT;
  int lo_all = 1 << 30, hi_all = -1;
  for (int x = 0; x < 2; ++x) {
    g.lo[x] = 1;
    g.hi[x] = 0;
    const int r0 = g.q0 + x * PPCfg::MT;
    const int r1 = min(p.Lq, r0 + PPCfg::MT) - 1;
    if (r0 > r1) continue;
    int lo0, hi0, lo1, hi1;
    visible_range(p, r0, lo0, hi0);
    visible_range(p, r1, lo1, hi1);
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

// Routing of key tile kt for both query tiles.
struct PPPlan {
  bool live[2];
  bool b16[2];   // bitmask: tile X is 16-bit
  bool need8, need16;
};

__device__ __forceinline__ PPPlan pp_plan(const AttnParams& p, const PPGeo& g, int kt) {
  PPPlan pl;
  const int c0 = kt * PPCfg::BN, c1 = min(p.Lk, c0 + PPCfg::BN) - 1;
  const int gi = kt / p.group_tiles;
  pl.need8 = pl.need16 = false;
  for (int x = 0; x < 2; ++x) {
    pl.live[x] = g.lo[x] <= g.hi[x] && g.lo[x] <= c1 && g.hi[x] >= c0 && kt >= 0;
    pl.b16[x] = false;
    if (!pl.live[x]) continue;
    if (p.adaptive) {
      pl.need8 = pl.need16 = true;
      continue;
    }
    int bit = 1;
    if (p.mask) {
      const int qt = 2 * g.pair + x;
      const size_t mi = (static_cast<size_t>(g.b * p.H + g.h) * p.nqt + qt) * p.mask_words + (gi >> 6);
      const uint64_t w = lamp_chk(mi < static_cast<size_t>(p.B) * p.H * p.nqt * p.mask_words, 1)
                             ? p.mask[mi] : ~0ull;
      bit = static_cast<int>((w >> (gi & 63)) & 1ull);
    }
    pl.b16[x] = (bit == 0);
    if (bit) pl.need8 = true; else pl.need16 = true;
  }
  return pl;
}

// ------------------------------------------------------------------ producer ----------

__device__ void pp_producer(const AttnParams& p, const PPGeo& g, uint8_t* smem, PPBars& bars,
                            const WaitCtx& wc) {
  using C = PPCfg;
  uint8_t* slots = smem + C::OFF_SLOTS;
  const int bh_q = g.b * p.H + g.h;
  const int bh_kv = g.b * p.Hkv + g.kvh;
  prefetch_tmap(&p.tm_q16);
  prefetch_tmap(&p.tm_k16);
  prefetch_tmap(&p.tm_v);
  prefetch_tmap(&p.tm_q8);
  prefetch_tmap(&p.tm_k8);
  if (!lamp_chk(bh_q < p.B * p.H && g.q0 < p.Lq + 2 * C::MT, 3)) return;
  mbar_arrive_expect_tx(&bars.q_full, 2 * (C::Q16_BYTES + C::Q8_BYTES));
  for (int x = 0; x < 2; ++x) {
    const int row = g.q0 + x * C::MT;
    for (int c = 0; c < 2; ++c)
      tma_load_3d(smem + C::OFF_Q16 + x * C::Q16_BYTES + c * C::MT * 128, &p.tm_q16, &bars.q_full,
                  c * 64, row, bh_q);
    tma_load_3d(smem + C::OFF_Q8 + x * C::Q8_BYTES, &p.tm_q8, &bars.q_full, 0, row, bh_q);
  }
  uint32_t item = 0;
  auto load = [&](int kind, int kt) -> bool {  // 0 K8, 1 K16, 2 V
    const int slot = static_cast<int>(item % C::NS);
    if (!lamp_chk(slot >= 0 && slot < C::NS && kt >= 0 && kt < p.nkt &&
                  bh_kv < p.B * p.Hkv, 2)) return false;
    const uint32_t use = item / C::NS;
    if (use > 0 && !mbar_wait(&bars.empty[slot], (use - 1) & 1u, wc, W_EMPTY)) return false;
    uint8_t* dst = slots + slot * C::SLOT_BYTES;
    const int row = kt * C::BN;
    if (kind == 0) {
      mbar_arrive_expect_tx(&bars.full[slot], C::BN * C::D);
      tma_load_3d(dst, &p.tm_k8, &bars.full[slot], 0, row, bh_kv);
    } else {
      const CUtensorMap* tm = (kind == 1) ? &p.tm_k16 : &p.tm_v;
      mbar_arrive_expect_tx(&bars.full[slot], C::BN * C::D * 2);
      tma_load_3d(dst, tm, &bars.full[slot], 0, row, bh_kv);
      tma_load_3d(dst + C::BN * 128, tm, &bars.full[slot], 64, row, bh_kv);
    }
    ++item;
    return true;
  };
  bool ok = true;
  for (int t = 0; ok && t < g.n; ++t) {
    const int kt = g.kt_lo + t;
    const PPPlan pl = pp_plan(p, g, kt);
    if (pl.need8 && !(ok = load(0, kt))) break;
    if (pl.need16 && !(ok = load(1, kt))) break;
    if (!(ok = load(2, kt))) break;
  }
  WaitCtx drain = wc;
  volatile uint32_t never = 0;
  drain.abort = &never;
  drain.limit_ns = 50000000ull;
  const uint32_t first = item > static_cast<uint32_t>(C::NS) ? item - C::NS : 0;
  for (uint32_t it = first; it < item; ++it)
    mbar_wait(&bars.full[it % C::NS], (it / C::NS) & 1u, drain, W_DRAIN);
  mbar_wait(&bars.q_full, 0, drain, W_DRAIN);
}

// ------------------------------------------------------------------ MMA issuer --------

__device__ void pp_mma(const AttnParams& p, const PPGeo& g, uint8_t* smem, PPBars& bars,
                       uint32_t tbase, const WaitCtx& wc) {
  using C = PPCfg;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t slots = sbase + C::OFF_SLOTS;
  const uint32_t f16 = p.bf16 ? 1u : 0u;
  const uint32_t id_s16 = idesc(1, f16, f16, 0, 0, C::BN, 128);
  // INT8 only: the host sends E4M3 work to the single-tile kernel (see lamp.cu).
  const uint32_t id_s8 = idesc(2, 1, 1, 0, 0, C::BN, 128);
  const uint32_t id_pv = idesc(1, f16, f16, 0, 1, C::D, 128);

  uint32_t item = 0;
  uint32_t cv[2] = {0, 0}, cp[2] = {0, 0};
  bool started[2] = {false, false};
  bool ok = mbar_wait(&bars.q_full, 0, wc, W_QFULL);
  tc_fence_after();

  // slots of the current / next key tile's items (-1 = not loaded)
  struct Items { int k8, k16, v; };
  auto take = [&](int& slot) -> bool {
    slot = static_cast<int>(item % C::NS);
    if (!lamp_chk(slot >= 0 && slot < C::NS, 4)) return false;
    const uint32_t use = item / C::NS;
    ++item;
    if (!mbar_wait(&bars.full[slot], use & 1u, wc, W_FULL)) return false;
    tc_fence_after();
    return true;
  };
  auto take_k = [&](const PPPlan& pl, Items& it) -> bool {
    it.k8 = it.k16 = it.v = -1;
    if (pl.need8 && !take(it.k8)) return false;
    if (pl.need16 && !take(it.k16)) return false;
    return true;
  };
  auto issue_s = [&](int x, bool sixteen, int slot) {
    const uint32_t dS = tbase + static_cast<uint32_t>(x * C::BN);
    const uint32_t ks = slots + slot * C::SLOT_BYTES;
    if (!lamp_chk(x >= 0 && x < 2 && slot >= 0 && slot < C::NS &&
                  ks + C::SLOT_BYTES <= sbase + C::OFF_BAR, 5)) return;
    if (sixteen) {
      const uint32_t qa = sbase + C::OFF_Q16 + x * C::Q16_BYTES;
#pragma unroll
      for (int s = 0; s < C::D / 16; ++s) {
        const int c = s >> 2, off = (s & 3) * 32;
        mma_f16_ss(dS, sdesc(qa + c * C::MT * 128 + off, 16, 1024, SWZ_128B),
                   sdesc(ks + c * C::BN * 128 + off, 16, 1024, SWZ_128B), id_s16, s > 0 ? 1u : 0u);
      }
    } else {
      const uint32_t qa = sbase + C::OFF_Q8 + x * C::Q8_BYTES;
#pragma unroll
      for (int s = 0; s < C::D / 32; ++s) {
        const uint64_t a = sdesc(qa + s * 32, 16, 1024, SWZ_128B);
        const uint64_t b = sdesc(ks + s * 32, 16, 1024, SWZ_128B);
        mma_i8_ss(dS, a, b, id_s8, s > 0 ? 1u : 0u);
      }
    }
  };
  auto first_s = [&](int x, const PPPlan& pl, const Items& it) {
    const bool sixteen = !p.adaptive && pl.b16[x];
    issue_s(x, sixteen, sixteen ? it.k16 : it.k8);
    tc_commit(&bars.s_full[x]);
  };

  Items cur{-1, -1, -1}, nxt{-1, -1, -1};
  PPPlan pl = pp_plan(p, g, g.kt_lo);
  if (ok && g.n > 0 && (ok = take_k(pl, cur))) {
    for (int x = 0; x < 2; ++x)
      if (pl.live[x]) first_s(x, pl, cur);
  }
  for (int t = 0; ok && t < g.n; ++t) {
    const int kt = g.kt_lo + t;
    const bool has_next = t + 1 < g.n;
    const PPPlan pn = has_next ? pp_plan(p, g, kt + 1) : PPPlan{};
    if (p.adaptive) {
      for (int x = 0; x < 2 && ok; ++x) {
        if (!pl.live[x]) continue;
        if (!(ok = mbar_wait(&bars.vote[x], cv[x] & 1u, wc, W_VOTE))) break;
        ++cv[x];
        tc_fence_after();
        const volatile uint32_t* vv = bars.votes[x];
        if ((vv[0] | vv[1] | vv[2] | vv[3]) != 0) {
          issue_s(x, true, cur.k16);
          tc_commit(&bars.s16_full[x]);
        }
      }
      if (!ok) break;
    }
    // every QK^T MMA of this key tile has been issued: release its K slots when they finish
    if (cur.k8 >= 0 && lamp_chk(cur.k8 < C::NS, 6)) tc_commit(&bars.empty[cur.k8]);
    if (cur.k16 >= 0 && lamp_chk(cur.k16 < C::NS, 6)) tc_commit(&bars.empty[cur.k16]);
    if (!(ok = take(cur.v))) break;
    const uint32_t vs = slots + cur.v * C::SLOT_BYTES;
    if (!(ok = lamp_chk(vs + C::SLOT_BYTES <= sbase + C::OFF_BAR, 7))) break;
    bool taken_next = false;
    for (int x = 0; x < 2; ++x) {
      if (pl.live[x]) {
        if (!(ok = mbar_wait(&bars.p_full[x], cp[x] & 1u, wc, W_PFULL))) break;
        ++cp[x];
        tc_fence_after();
        const uint32_t pt = tbase + static_cast<uint32_t>(x * C::BN);
        const uint32_t ot = tbase + static_cast<uint32_t>(2 * C::BN + x * C::D);
#pragma unroll
        for (int s = 0; s < C::BN / 16; ++s) {
          const uint64_t b = sdesc(vs + s * 16 * 128, C::BN * 128, 1024, SWZ_128B);
          mma_f16_ts(ot, pt + s * 8, b, id_pv, (started[x] || s > 0) ? 1u : 0u);
        }
        started[x] = true;
      }
      if (has_next && pn.live[x]) {
        if (!taken_next) {
          if (!(ok = take_k(pn, nxt))) break;
          taken_next = true;
        }
        first_s(x, pn, nxt);
      }
    }
    if (!ok) break;
    if (lamp_chk(cur.v >= 0 && cur.v < C::NS, 8)) tc_commit(&bars.empty[cur.v]);
    cur = nxt;
    pl = pn;
  }
  tc_commit(&bars.o_done[0]);
  tc_commit(&bars.o_done[1]);
  tc_commit(&bars.drain);
  WaitCtx drain = wc;
  volatile uint32_t never = 0;
  drain.abort = &never;
  drain.limit_ns = 50000000ull;
  mbar_wait(&bars.drain, 0, drain, W_DRAIN);
}

// ------------------------------------------------------------------ softmax -----------

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// One row per thread.  Per key tile: read S from TMEM, turn it into fp32 scores of the raw
// product (exact int32 -> fp32 for 8-bit tiles), mask, take the row max, vote (look-ahead
// rule), exponentiate against the lazy reference max, pack P as 16-bit pairs into the S
// columns, and keep the two row sums: of the exact p (for lse) and of the rounded p that the
// P.V MMA multiplies (for O).
template <bool BF16>
__device__ void pp_softmax(const AttnParams& p, const PPGeo& g, PPBars& bars, uint32_t tbase,
                           const WaitCtx& wc) {
  using C = PPCfg;
  const int x = threadIdx.x >> 7;            // query tile of this warpgroup
  const int warp = (threadIdx.x >> 5) & 3;   // TMEM lane quadrant
  const int lane = threadIdx.x & 31;
  const int r = warp * 32 + lane;
  const int i = g.q0 + x * C::MT + r;
  const bool row_valid = i < p.Lq;
  const int qt = 2 * g.pair + x;
  const int bh_q = g.b * p.H + g.h;
  const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
  const uint32_t s_col = static_cast<uint32_t>(x * C::BN);
  const uint32_t o_col = static_cast<uint32_t>(2 * C::BN + x * C::D);
  int lo_r = 1, hi_r = 0;
  if (row_valid) visible_range(p, i, lo_r, hi_r);
  const float sq = (row_valid && qt < p.nqt &&
                    lamp_chk(static_cast<size_t>(bh_q) * p.nqt + qt < static_cast<size_t>(p.B) * p.H * p.nqt, 9))
                       ? __ldg(p.q_scale + static_cast<size_t>(bh_q) * p.nqt + qt) : 0.0f;
  const float* ks_row = p.k_scale + static_cast<size_t>(g.b * p.Hkv + g.kvh) * p.nkt;
  const float NEG_INF = -__int_as_float(0x7f800000);
  const float sq_scale = sq * p.scale_log2;

  float m_ref = NEG_INF;   // max used for the exponentials (lazy)
  float m_true = NEG_INF;  // true running max of the used scores (look-ahead rule)
  float l_ex = 0.0f, l_rd = 0.0f;
  uint32_t cs = 0, c16 = 0, cvv = 0;
  bool ok = true, any_pv = false;
  uint32_t raw[C::BN];

  auto load_s = [&]() {
#pragma unroll
    for (int c = 0; c < C::BN / 32; ++c)
      tmem_ld32(lane_base + s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
    tmem_wait_ld();
  };
  // int32 accumulators -> exact fp32 (|acc| < 2^22): (acc + 1.5*2^23 as bits) - 1.5*2^23
  auto int_to_float = [&]() {
#pragma unroll
    for (int c = 0; c < C::BN; c += 2) {
      const uint64_t v = f2_add(f2_pack(__uint_as_float(raw[c] + 0x4B400000u),
                                        __uint_as_float(raw[c + 1] + 0x4B400000u)),
                                f2_pack(-12582912.0f, -12582912.0f));
      float a, b;
      f2_unpack(v, a, b);
      raw[c] = __float_as_uint(a);
      raw[c + 1] = __float_as_uint(b);
    }
  };
  // keep columns [a, b] of the tile (the row's visible keys), -inf elsewhere; branch-free
  auto apply_mask = [&](int j0) {
    const int a = row_valid ? lo_r - j0 : C::BN;
    const int b = row_valid ? hi_r - j0 : -1;
#pragma unroll
    for (int c = 0; c < C::BN; ++c) raw[c] = (c < a || c > b) ? 0xff800000u : raw[c];
  };
  auto raw_max = [&]() -> float {
    float m0 = NEG_INF, m1 = NEG_INF, m2 = NEG_INF, m3 = NEG_INF;
#pragma unroll
    for (int c = 0; c < C::BN; c += 8) {
      m0 = max3(m0, __uint_as_float(raw[c]), __uint_as_float(raw[c + 1]));
      m1 = max3(m1, __uint_as_float(raw[c + 2]), __uint_as_float(raw[c + 3]));
      m2 = max3(m2, __uint_as_float(raw[c + 4]), __uint_as_float(raw[c + 5]));
      m3 = max3(m3, __uint_as_float(raw[c + 6]), __uint_as_float(raw[c + 7]));
    }
    return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  };

  // scalars of the next live tile are fetched one tile ahead (off the critical path)
  int t_next = 0;
  while (t_next < g.n && !pp_plan(p, g, g.kt_lo + t_next).live[x]) ++t_next;
  PPPlan pl_n = pp_plan(p, g, g.kt_lo + min(t_next, g.n - 1));
  float ks_n = (t_next < g.n) ? __ldg(ks_row + g.kt_lo + t_next) : 0.0f;

  while (ok && t_next < g.n) {
    const int t = t_next;
    const int kt = g.kt_lo + t;
    const PPPlan pl = pl_n;
    const float ks = ks_n;
    ++t_next;
    while (t_next < g.n && !pp_plan(p, g, g.kt_lo + t_next).live[x]) ++t_next;
    if (t_next < g.n) {
      pl_n = pp_plan(p, g, g.kt_lo + t_next);
      ks_n = __ldg(ks_row + g.kt_lo + t_next);
    }

    if (!(ok = warp_wait(&bars.s_full[x], cs & 1u, wc, W_SFULL))) break;
    ++cs;
    tc_fence_after();
    load_s();
    const int j0 = kt * C::BN;
    const bool full = row_valid && j0 >= lo_r && j0 + C::BN - 1 <= hi_r;
    bool sixteen = !p.adaptive && pl.b16[x];
    // (a zero block scale would turn masked -inf entries into NaN: keep it positive; the
    // scores of an all-zero block are 0 either way)
    float cscale = sixteen ? p.scale_log2 : fmaxf(sq_scale * ks, 1e-30f);
    if (!sixteen) int_to_float();
    if (!full) apply_mask(j0);
    float tmax = raw_max();
    bool flagged = false;
    if (p.adaptive) {
      const float t8 = (tmax == NEG_INF) ? NEG_INF : tmax * cscale;
      const bool vote = (t8 != NEG_INF) && (t8 >= m_true - p.tau_log2);
      const uint32_t wv = __any_sync(0xFFFFFFFFu, vote) ? 1u : 0u;
      if (lane == 0) bars.votes[x][warp] = wv;
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
        sixteen = true;
        cscale = p.scale_log2;
        if (!full) apply_mask(j0);
        tmax = raw_max();
      }
    }
    if (p.route && lane == 0 && warp == 0 &&
        lamp_chk((static_cast<size_t>(bh_q) * p.nqt + qt) * p.nkt + kt <
                     static_cast<size_t>(p.B) * p.H * p.nqt * p.nkt && qt < p.nqt, 11))
      p.route[(static_cast<size_t>(bh_q) * p.nqt + qt) * p.nkt + kt] =
          p.adaptive ? (flagged ? 3 : 1) : (sixteen ? 2 : 1);

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

    // p = 2^(value * cscale - m_ref); masked entries hold -inf and give 0
    const float mu = (m_ref == NEG_INF) ? 0.0f : m_ref;
    const uint64_t c2 = f2_pack(cscale, cscale);
    const uint64_t nb2 = f2_pack(-mu, -mu);
    uint64_t se0 = 0, se1 = 0, sr0 = 0, sr1 = 0;
#pragma unroll
    for (int c = 0; c < C::BN; c += 2) {
      float x0, x1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), c2, nb2),
                x0, x1);
      const float p0 = ex2(x0), p1 = ex2(x1);
      uint32_t pk;
      float r0, r1;
      if (BF16) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk = *reinterpret_cast<uint32_t*>(&h2);
        r0 = __uint_as_float(pk << 16);
        r1 = __uint_as_float(pk & 0xFFFF0000u);
      } else {
        __half2 h2 = __floats2half2_rn(p0, p1);
        pk = *reinterpret_cast<uint32_t*>(&h2);
        r0 = __low2float(h2);
        r1 = __high2float(h2);
      }
      if (c & 2) {
        se1 = f2_add(se1, f2_pack(p0, p1));
        sr1 = f2_add(sr1, f2_pack(r0, r1));
      } else {
        se0 = f2_add(se0, f2_pack(p0, p1));
        sr0 = f2_add(sr0, f2_pack(r0, r1));
      }
      raw[c >> 1] = pk;
    }
    {
      float a0, a1, b0, b1;
      f2_unpack(f2_add(se0, se1), a0, a1);
      f2_unpack(f2_add(sr0, sr1), b0, b1);
      l_ex += a0 + a1;
      l_rd += b0 + b1;
    }
#pragma unroll
    for (int c = 0; c < C::BN / 32; ++c) tmem_st16(lane_base + s_col + c * 16, &raw[c * 16]);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.p_full[x]);
    any_pv = true;
  }
  if (!ok) return;

  if (any_pv) {
    if (!warp_wait(&bars.o_done[x], 0, wc, W_ODONE)) return;
    tc_fence_after();
  }
  const float inv = (l_rd > 0.0f) ? 1.0f / l_rd : 0.0f;
  const size_t orow = (static_cast<size_t>(bh_q) * p.Lq + (row_valid ? i : 0)) * C::D;
#pragma unroll 1
  for (int c = 0; c < C::D / 32; ++c) {
    uint32_t ov[32];
    if (any_pv) {
      tmem_ld32(lane_base + o_col + c * 32, ov);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] = 0u;
    }
    if (!row_valid) continue;
    if (!lamp_chk(orow + c * 32 + 32 <= static_cast<size_t>(p.B) * p.H * p.Lq * C::D, 12)) continue;
    if (p.out_f32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + c * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                             __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow + c * 32);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = __uint_as_float(ov[8 * e + 2 * q]) * inv;
          const float b2 = __uint_as_float(ov[8 * e + 2 * q + 1]) * inv;
          if (BF16) {
            __nv_bfloat162 v2 = __floats2bfloat162_rn(a, b2);
            w[q] = *reinterpret_cast<uint32_t*>(&v2);
          } else {
            __half2 v2 = __floats2half2_rn(a, b2);
            w[q] = *reinterpret_cast<uint32_t*>(&v2);
          }
        }
        dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  if (row_valid && p.lse &&
      lamp_chk(static_cast<size_t>(bh_q) * p.Lq + i < static_cast<size_t>(p.B) * p.H * p.Lq, 13))
    p.lse[static_cast<size_t>(bh_q) * p.Lq + i] =
        (l_ex > 0.0f) ? m_ref * 0.69314718055994530942f + logf(l_ex) : NEG_INF;
}

// ------------------------------------------------------------------ kernel ------------

template <bool BF16>
__global__ void __launch_bounds__(384, 1) attn_fwd_pp_kernel(const __grid_constant__ AttnParams p) {
  using C = PPCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  PPBars& bars = *reinterpret_cast<PPBars*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5;
  const PPGeo g = pp_geo(p);
  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.s16_full[x], 1);
      mbar_init(&bars.vote[x], 4);
      mbar_init(&bars.p_full[x], 4);
      mbar_init(&bars.o_done[x], 1);
    }
    mbar_init(&bars.drain, 1);
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
  WaitCtx wc{&bars.abort, &g_lamp_error, p.wait_ns};
  // Register split within the launch allotment of 384 x 168: the producer / MMA warpgroup
  // gives back to 120 per thread, the two softmax warpgroups grow to 192
  // (128 * 120 + 256 * 192 = 64512 = 384 * 168).
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    pp_softmax<BF16>(p, g, bars, tbase, wc);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;\n" ::: "memory");
    if (warp == 8) {
      if ((threadIdx.x & 31) == 0 && g.n > 0) pp_producer(p, g, smem, bars, wc);
    } else if (warp == 9) {
      if ((threadIdx.x & 31) == 0 && g.n > 0) pp_mma(p, g, smem, bars, tbase, wc);
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
