// CPU oracle for tile-routed mixed-precision attention (prefill forward).
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this file;
// only the tests, the smoke check and the benchmark's CPU-baseline leg use it.  It shares no
// code, header, table or constant with the CUDA library.
//
// Plain and slow on purpose: loops over rows, keys and channels; exact integer dot products
// for INT8 tiles, exact fp64 sums for E4M3 tiles (every product of two e4m3 codes is exact in
// fp64 and the sums stay far below 2^53), fp64 dot products on the 16-bit inputs for 16-bit
// tiles, and a two-pass fp64 softmax.  Sources:
//   * TileMix page, section 2 "How It Works", "The Dual-Path Engine": INT8 path = per-block
//     quantised Q and K, tensor-core product, rescale with per-block scale factors; FP16 path =
//     plain floating-point product; both feed one shared online-softmax state.
//   * TileMix page, section 2, "Packed Bitmasks": one bit per group of adjacent key tiles,
//     0 = FP16, 1 = INT8, one mask per query row (read here: per query routing tile).
//   * LampAttention page, abstract: 8-bit key-query products, sensitive sub-blocks found
//     adaptively and recomputed in 16 bits.  The rule used: a tile is recomputed when, for some
//     row, its 8-bit tile max reaches the running row max minus tau.
// Readings of the pages that they leave open are listed with each function below.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------------------
// E4M3 (OCP "e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits, no infinities,
// S.1111.111 is NaN, largest finite 448, subnormals 2^-6 * m/8.
// ---------------------------------------------------------------------------------------
double e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// Round to nearest representable e4m3 value, ties to even mantissa, saturating to +-448.
uint8_t e4m3_encode(float xf) {
  double x = xf;
  if (std::isnan(x)) return 0x7F;
  uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(x);
  if (a >= 448.0) return sign | 0x7E;  // satfinite (RNE of [448,464) is 448 as well)
  const double min_normal = std::ldexp(1.0, -6);
  if (a < min_normal) {
    // subnormal grid: multiples of 2^-9
    double qm = std::nearbyint(a * 512.0);  // exact scaling, RNE
    int m = (int)qm;                        // 0..8; 8 is the smallest normal (code 0x08)
    return sign | (uint8_t)m;
  }
  int E;
  std::frexp(a, &E);          // a = f * 2^E, f in [0.5, 1)
  int e = E - 1;              // a = mant * 2^e, mant in [1, 2)
  double mant = std::ldexp(a, -e);
  double qm = std::nearbyint((mant - 1.0) * 8.0);  // exact, RNE
  int m = (int)qm;
  if (m == 8) { m = 0; e += 1; }
  int code = ((e + 7) << 3) | m;
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

// ---------------------------------------------------------------------------------------
// Per-block quantisation (TileMix "Dual-Path Engine", INT8 path; LampAttention 8-bit formats).
// Block = `blk` consecutive rows x all D channels of one (batch, head).  Reading: the block
// is the routing tile's extent on that operand; scale = absmax / 127 (INT8, symmetric, codes
// in [-127, 127]) or absmax / 448 (E4M3); codes = round-to-nearest-even of x / scale, both the
// scale and the quotient rounded to fp32 (IEEE divide); an all-zero block has scale 0, codes 0.
// ---------------------------------------------------------------------------------------
void quantize_block(const float* x, int rows, int D, int fmt, uint8_t* codes, float* scale) {
  float a = 0.0f;
  for (int r = 0; r < rows; ++r)
    for (int d = 0; d < D; ++d) a = std::fmax(a, std::fabs(x[(size_t)r * D + d]));
  if (a == 0.0f) {
    *scale = 0.0f;
    std::memset(codes, 0, (size_t)rows * D);
    return;
  }
  const float denom = (fmt == 0) ? 127.0f : 448.0f;
  float s = a / denom;  // IEEE fp32 divide (the build forbids contraction and fast-math)
  *scale = s;
  for (int r = 0; r < rows; ++r)
    for (int d = 0; d < D; ++d) {
      float y = x[(size_t)r * D + d] / s;
      if (fmt == 0) {
        float c = std::nearbyint(y);
        if (c > 127.0f) c = 127.0f;
        if (c < -127.0f) c = -127.0f;
        codes[(size_t)r * D + d] = (uint8_t)(int8_t)(int)c;
      } else {
        codes[(size_t)r * D + d] = e4m3_encode(y);
      }
    }
}

// ---------------------------------------------------------------------------------------
// 8-bit exponentials and 8-bit P.V (LampAttention page, abstract: the exponentials are
// evaluated in 8-bit formats; the pages fix no format, so the reading is E4M3 for both P and
// V).
//
// V: one scale per (batch, KV head, channel) over all keys of the plane (the pages give no V
// block; a per-channel scale commutes with the sum over keys, so it applies to O once):
// a = max_j |v_jd|, s = fl32(a / 448), code = E4M3(fl32(v / s)) rounded to nearest even,
// saturating; a = 0 gives s = 0 and zero codes.  Codes are laid out [D][Lk] (channel-major).
// ---------------------------------------------------------------------------------------
void quantize_v_plane(const float* v, int Lk, int D, uint8_t* codes_t, float* scales) {
  for (int d = 0; d < D; ++d) {
    float a = 0.0f;
    for (int j = 0; j < Lk; ++j) a = std::fmax(a, std::fabs(v[(size_t)j * D + d]));
    const float s = a / 448.0f;  // IEEE fp32 divide
    scales[d] = (a == 0.0f) ? 0.0f : s;
    for (int j = 0; j < Lk; ++j)
      codes_t[(size_t)d * Lk + j] = (a == 0.0f) ? 0 : e4m3_encode(v[(size_t)j * D + d] / s);
  }
}

// P: the nearest E4M3 value of a non-negative p <= 448 (ties to even), computed from the
// format's grid (a step of 2^-9 below 2^-6, else 2^(e-3) on [2^e, 2^(e+1))), and the relative
// distance of p from the nearest rounding midpoint: how far p is from rounding the other way.
double e4m3_round_pos(double p, double* midpoint_dist) {
  if (!(p > 0.0)) {
    if (midpoint_dist) *midpoint_dist = std::numeric_limits<double>::infinity();
    return 0.0;
  }
  double step;
  if (p < 0.015625) {
    step = 0.001953125;
  } else {
    int E;
    std::frexp(p, &E);  // p in [2^(E-1), 2^E)
    step = std::ldexp(1.0, E - 1 - 3);
  }
  const double q = p / step;  // exact: step is a power of two
  const double fl = std::floor(q), frac = q - fl;
  double n;
  if (frac > 0.5) n = fl + 1.0;
  else if (frac < 0.5) n = fl;
  else n = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  if (midpoint_dist) *midpoint_dist = std::fabs(frac - 0.5) * step / p;
  return n * step;
}

// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014): one step of the generator from state x:
// add the golden gamma, then the variant-13 finaliser.
uint64_t splitmix64_next(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

struct Geometry {
  int B, H, Hkv, Lq, Lk, D, bm, bn, causal, window;
  int nqt() const { return (Lq + bm - 1) / bm; }
  int nkt() const { return (Lk + bn - 1) / bn; }
  // Reading (causal, bottom-right aligned; window of W keys including the diagonal):
  // query i sees key j iff j <= i + (Lk - Lq) and, when W > 0, j > i + (Lk - Lq) - W.
  void visible(int i, long* lo, long* hi) const {
    if (!causal) { *lo = 0; *hi = Lk - 1; return; }
    long h = (long)i + (Lk - Lq);
    if (h > Lk - 1) h = Lk - 1;
    long l = 0;
    if (window > 0) { l = (long)i + (Lk - Lq) - window + 1; if (l < 0) l = 0; }
    *lo = l; *hi = h;
  }
};

}  // namespace

extern "C" {

struct orc_args {
  const float* q;      // [B,H,Lq,D]   exact values of the 16-bit inputs
  const float* k;      // [B,Hkv,Lk,D]
  const float* v;      // [B,Hkv,Lk,D]
  int B, H, Hkv, Lq, Lk, D, bm, bn;
  int causal, window;
  double scale;            // softmax scale applied to q.k
  const uint64_t* mask;    // bitmask routing [B,H,nQT,W] (NULL: every tile 8-bit)
  int mask_words;          // W
  int group_tiles;
  int adaptive;            // 0: bitmask routing, 1: look-ahead rule
  int fmt;                 // 0: INT8, 1: E4M3
  double tau;
  const int64_t* rows;     // optional [B,H,nrows] sorted query rows; NULL = every row
  int nrows;
  int threads;
  double* o;               // [B,H,R,D]  R = nrows or Lq
  double* lse;             // [B,H,R]
  uint8_t* route;          // optional [B,H,nQT,nKT]: 0 dead, 1 8-bit, 2 16-bit by mask, 3 16-bit flagged,
                           // 4 dropped by the threshold skip
  double* margin;          // optional [B,H,nQT,nKT]: adaptive decision margin (inf elsewhere)
  const uint8_t* route_hint;  // optional [B,H,nQT,nKT]: decisions to follow where margin < hint_margin
  double hint_margin;
  uint8_t* q_codes;        // optional [B,H,Lq,D] output of the Q quantiser (all blocks)
  float* q_scales;         // optional [B,H,nQT]
  uint8_t* k_codes;        // optional [B,Hkv,Lk,D]
  float* k_scales;         // optional [B,Hkv,nKT]
  double skip_tau;         // look-ahead mode: drop a tile every row of which is this far below
                           // its running max (+inf: never)
  // optional: 8-bit K given instead of quantised here (an 8-bit key cache, TileMix page,
  // section 4: INT8 key/value caches for decode); the 8-bit path then uses these codes and
  // scales, the 16-bit path the values in k
  const uint8_t* k_codes_in;  // [B,Hkv,Lk,D]
  const float* k_scales_in;   // [B,Hkv,nKT]
  uint8_t* hinted;            // optional [B,H,nQT,nKT]: 1 where a decision followed route_hint
                              // against the rule's own outcome (its margin < hint_margin)
  // 8-bit exponentials and 8-bit P.V (see e4m3_round_pos and quantize_v_plane): O of a row is
  // sv * sum_t 2^(m_t - m) sum_{j in t} p8_j v8_j / sum_t 2^(m_t - m) sum_{j in t} p8_j, with
  // key tiles t in ascending order, m_t the row's running max of the routed scores after tile
  // t, m the final one, and p8_j = E4M3(e^(s_j - m_t) * 2^8) (the largest p is 256 < 448).
  // lse stays the exact softmax's.
  int pv8;
  uint8_t* v_codes;           // optional [B,Hkv,D,Lk] output of the V quantiser
  float* v_scales;            // optional [B,Hkv,D]
  double* pv8_margin;         // optional [B,H,R]: the row's smallest midpoint distance of a p
};

double orc_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
double orc_e4m3_round_pos(double p, double* midpoint_dist) { return e4m3_round_pos(p, midpoint_dist); }
// Per-channel 8-bit V of x [outer, Lk, D]: codes [outer, D, Lk], scales [outer, D].
void orc_quantize_v(const float* x, int outer, int Lk, int D, uint8_t* codes_t, float* scales) {
  for (int o = 0; o < outer; ++o)
    quantize_v_plane(x + (size_t)o * Lk * D, Lk, D, codes_t + (size_t)o * D * Lk,
                     scales + (size_t)o * D);
}
uint8_t orc_e4m3_encode(float x) { return e4m3_encode(x); }
uint64_t orc_splitmix64_next(uint64_t x) { return splitmix64_next(x); }

// Quantise x [outer, L, D] in blocks of `blk` rows: codes [outer, L, D], scales [outer, ceil(L/blk)].
void orc_quantize(const float* x, int outer, int L, int D, int blk, int fmt, uint8_t* codes,
                  float* scales) {
  int nb = (L + blk - 1) / blk;
  for (int o = 0; o < outer; ++o)
    for (int b = 0; b < nb; ++b) {
      int r0 = b * blk, rows = (L - r0 < blk) ? (L - r0) : blk;
      size_t off = ((size_t)o * L + r0) * D;
      quantize_block(x + off, rows, D, fmt, codes + off, scales + (size_t)o * nb + b);
    }
}

// Seeded Bernoulli routing template (the pages' routing policy is a static, data-free
// template; the exact template shape is not given, so each group bit is drawn i.i.d.):
// bit g of the mask of (b, h, qt) is 0 (16-bit) iff u53 * 2^-53 < p_fp16, where
// u = splitmix64_next(seed XOR idx * 0x9E3779B97F4A7C15), idx = ((b*H + h)*nQT + qt)*nG + g
// and u53 = u >> 11.  Bits at g >= nG are zero.
void orc_build_mask(uint64_t* mask, int B, int H, int nqt, int ng, int W, double p_fp16,
                    uint64_t seed) {
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int qt = 0; qt < nqt; ++qt) {
        uint64_t* row = mask + (((size_t)b * H + h) * nqt + qt) * W;
        for (int w = 0; w < W; ++w) row[w] = 0;
        for (int g = 0; g < ng; ++g) {
          uint64_t idx = (((uint64_t)b * H + h) * nqt + qt) * (uint64_t)ng + g;
          uint64_t u = splitmix64_next(seed ^ (idx * 0x9E3779B97F4A7C15ull));
          double r = (double)(u >> 11) * 0x1.0p-53;
          int eight_bit = (r < p_fp16) ? 0 : 1;
          if (eight_bit) row[g >> 6] |= (1ull << (g & 63));
        }
      }
}

// Structured static routing template (TileMix page, section 4 "Why It Matters": the routing
// policy is a static, data-free structured template; section 3: the "SpTrans75" configuration
// routes 75% of the work to INT8).  The pages give no shape; the reading used, after the
// strided and local layouts of sparse transformers: for the routing row qt, the diagonal key
// tile kd holds the key aligned with the row's last query, min(Lq, (qt+1) BM) - 1 + Lk - Lq
// (bottom-right), clamped to [0, nKT - 1]; gd = kd / group_tiles is its group.  Group g is
// FP16 (bit 0) iff g < sink, or |gd - g| < band, or stride > 0 and |gd - g| is a multiple of
// stride; every other group is INT8 (bit 1).  Bits at g >= nG are zero.
void orc_build_mask_template(uint64_t* mask, int B, int H, int Lq, int Lk, int bm, int bn,
                             int group_tiles, int sink, int band, int stride) {
  const int nqt = (Lq + bm - 1) / bm, nkt = (Lk + bn - 1) / bn;
  const int ng = (nkt + group_tiles - 1) / group_tiles;
  const int W = (ng + 63) / 64 > 0 ? (ng + 63) / 64 : 1;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int qt = 0; qt < nqt; ++qt) {
        uint64_t* row = mask + (((size_t)b * H + h) * nqt + qt) * W;
        for (int w = 0; w < W; ++w) row[w] = 0;
        long last_q = std::min<long>(Lq, (long)(qt + 1) * bm) - 1;
        long kd = (last_q + Lk - Lq) / bn;
        if (last_q + Lk - Lq < 0) kd = 0;
        if (kd > nkt - 1) kd = nkt - 1;
        const long gd = kd / group_tiles;
        for (int g = 0; g < ng; ++g) {
          const long d = std::labs(gd - g);
          const bool fp16 = g < sink || d < band || (stride > 0 && d % stride == 0);
          if (!fp16) row[g >> 6] |= (1ull << (g & 63));
        }
      }
}

// Raw score tiles (the reference of the library's debug capture).  For each listed routing tile
// (b, h, qt, kt) -- tiles[4 * t + 0..3] -- the unscaled product over every position of the tile,
// query row i = qt * bm + r and key j = kt * bn + c, with rows or keys past the problem counting
// as zero vectors (the 8-bit product is what the scores of TileMix's INT8 path are made of,
// before the rescale with the two block scales):
//   kind 0: sum_d cq[i][d] * ck[j][d] over INT8 codes, exact int64;
//   kind 1: the same over E4M3 codes, each decoded exactly, summed in fp64 (every product is
//           exact and the sums stay far below 2^53, so the sum is exact);
//   kind 2: sum_d q[i][d] * k[j][d] over the 16-bit inputs' values, in fp64.
// qx / kx: uint8 codes (kinds 0, 1) or fp32 values (kind 2), [B][H][Lq][D] and [B][Hkv][Lk][D];
// query head h reads KV head h / (H / Hkv).  out: fp64 [n][bm][bn].  Returns 1 on bad arguments.
int orc_score_tiles(const void* qx, const void* kx, int B, int H, int Hkv, int Lq, int Lk, int D,
                    int bm, int bn, int kind, const int32_t* tiles, int n, double* out) {
  if (H % Hkv != 0 || kind < 0 || kind > 2) return 1;
  const int G = H / Hkv;
  for (int t = 0; t < n; ++t) {
    const int b = tiles[4 * t], h = tiles[4 * t + 1], qt = tiles[4 * t + 2], kt = tiles[4 * t + 3];
    if (b < 0 || b >= B || h < 0 || h >= H || qt < 0 || kt < 0) return 1;
    const int kvh = h / G;
    for (int r = 0; r < bm; ++r)
      for (int c = 0; c < bn; ++c) {
        const long i = (long)qt * bm + r, j = (long)kt * bn + c;
        double v = 0.0;
        if (i < Lq && j < Lk) {
          const size_t qo = (((size_t)b * H + h) * Lq + i) * D;
          const size_t ko = (((size_t)b * Hkv + kvh) * Lk + j) * D;
          if (kind == 0) {
            const uint8_t* cq = static_cast<const uint8_t*>(qx) + qo;
            const uint8_t* ck = static_cast<const uint8_t*>(kx) + ko;
            int64_t acc = 0;
            for (int d = 0; d < D; ++d) acc += (int64_t)(int8_t)cq[d] * (int64_t)(int8_t)ck[d];
            v = (double)acc;
          } else if (kind == 1) {
            const uint8_t* cq = static_cast<const uint8_t*>(qx) + qo;
            const uint8_t* ck = static_cast<const uint8_t*>(kx) + ko;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += e4m3_decode(cq[d]) * e4m3_decode(ck[d]);
            v = acc;
          } else {
            const float* x = static_cast<const float*>(qx) + qo;
            const float* y = static_cast<const float*>(kx) + ko;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += (double)x[d] * (double)y[d];
            v = acc;
          }
        }
        out[((size_t)t * bm + r) * bn + c] = v;
      }
  }
  return 0;
}

int orc_attention(const orc_args* a) {
  Geometry g{a->B, a->H, a->Hkv, a->Lq, a->Lk, a->D, a->bm, a->bn, a->causal, a->window};
  if (g.H % g.Hkv != 0 || g.D <= 0 || g.bm <= 0 || g.bn <= 0) return 1;
  const int G = g.H / g.Hkv, D = g.D, nqt = g.nqt(), nkt = g.nkt();
  const double NEG_INF = -std::numeric_limits<double>::infinity();
  const double INF = std::numeric_limits<double>::infinity();

  // Quantise K for every (b, kv head) block of bn rows.
  std::vector<uint8_t> kc((size_t)g.B * g.Hkv * g.Lk * D);
  std::vector<float> ks((size_t)g.B * g.Hkv * nkt);
  if (a->k_codes_in && a->k_scales_in) {
    std::memcpy(kc.data(), a->k_codes_in, kc.size());
    std::memcpy(ks.data(), a->k_scales_in, ks.size() * sizeof(float));
  } else {
    orc_quantize(a->k, g.B * g.Hkv, g.Lk, D, g.bn, a->fmt, kc.data(), ks.data());
  }
  // 8-bit V, per channel (8-bit P.V only)
  std::vector<uint8_t> vc;
  std::vector<float> vs;
  if (a->pv8) {
    vc.resize((size_t)g.B * g.Hkv * D * g.Lk);
    vs.resize((size_t)g.B * g.Hkv * D);
    for (int p = 0; p < g.B * g.Hkv; ++p)
      quantize_v_plane(a->v + (size_t)p * g.Lk * D, g.Lk, D, vc.data() + (size_t)p * D * g.Lk,
                       vs.data() + (size_t)p * D);
    if (a->v_codes) std::memcpy(a->v_codes, vc.data(), vc.size());
    if (a->v_scales) std::memcpy(a->v_scales, vs.data(), vs.size() * sizeof(float));
  }
  if (a->k_codes) std::memcpy(a->k_codes, kc.data(), kc.size());
  if (a->k_scales) std::memcpy(a->k_scales, ks.data(), ks.size() * sizeof(float));
  if (a->q_codes || a->q_scales) {
    std::vector<uint8_t> qc((size_t)g.B * g.H * g.Lq * D);
    std::vector<float> qs((size_t)g.B * g.H * nqt);
    orc_quantize(a->q, g.B * g.H, g.Lq, D, g.bm, a->fmt, qc.data(), qs.data());
    if (a->q_codes) std::memcpy(a->q_codes, qc.data(), qc.size());
    if (a->q_scales) std::memcpy(a->q_scales, qs.data(), qs.size() * sizeof(float));
  }

  // Work items: (b, h, qt) tiles that hold at least one requested row.
  const int R = a->rows ? a->nrows : g.Lq;
  struct Item { int b, h, qt, r_begin, r_end; };  // [r_begin, r_end) into the requested rows
  std::vector<Item> items;
  for (int b = 0; b < g.B; ++b)
    for (int h = 0; h < g.H; ++h) {
      if (!a->rows) {
        for (int qt = 0; qt < nqt; ++qt) {
          int r0 = qt * g.bm, r1 = std::min(g.Lq, r0 + g.bm);
          items.push_back({b, h, qt, r0, r1});
        }
      } else {
        const int64_t* rr = a->rows + ((size_t)b * g.H + h) * R;
        int s = 0;
        while (s < R) {
          int qt = (int)(rr[s] / g.bm), e = s;
          while (e < R && rr[e] / g.bm == qt) ++e;
          items.push_back({b, h, qt, s, e});
          s = e;
        }
      }
    }
  if (a->route) std::memset(a->route, 0, (size_t)g.B * g.H * nqt * nkt);
  if (a->hinted) std::memset(a->hinted, 0, (size_t)g.B * g.H * nqt * nkt);
  if (a->margin)
    for (size_t i = 0; i < (size_t)g.B * g.H * nqt * nkt; ++i) a->margin[i] = INF;

  std::atomic<size_t> next{0};
  auto worker = [&]() {
    std::vector<uint8_t> qcode((size_t)g.bm * D);
    std::vector<double> m_run(g.bm), s8row(g.bn), s16row(g.bn);
    std::vector<uint8_t> tile_route(nkt);
    std::vector<double> srow(g.Lk);
    for (;;) {
      size_t it = next.fetch_add(1);
      if (it >= items.size()) break;
      const Item& I = items[it];
      const int b = I.b, h = I.h, qt = I.qt, kvh = h / G;
      const int r0 = qt * g.bm, rows_in_tile = std::min(g.Lq, r0 + g.bm) - r0;
      const float* qh = a->q + ((size_t)b * g.H + h) * g.Lq * D;
      const float* kh = a->k + ((size_t)b * g.Hkv + kvh) * g.Lk * D;
      const float* vh = a->v + ((size_t)b * g.Hkv + kvh) * g.Lk * D;
      const uint8_t* kch = kc.data() + ((size_t)b * g.Hkv + kvh) * g.Lk * D;
      const float* ksh = ks.data() + ((size_t)b * g.Hkv + kvh) * nkt;
      float qscale;
      quantize_block(qh + (size_t)r0 * D, rows_in_tile, D, a->fmt, qcode.data(), &qscale);

      // 8-bit score of (query row r0+r, key j): exact code dot product times the scales.
      auto score8 = [&](int r, long j) -> double {
        const uint8_t* cq = qcode.data() + (size_t)r * D;
        const uint8_t* ck = kch + (size_t)j * D;
        double dot;
        if (a->fmt == 0) {
          int64_t acc = 0;
          for (int d = 0; d < D; ++d) acc += (int64_t)(int8_t)cq[d] * (int64_t)(int8_t)ck[d];
          dot = (double)acc;
        } else {
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += e4m3_decode(cq[d]) * e4m3_decode(ck[d]);
          dot = acc;
        }
        int kt = (int)(j / g.bn);
        return dot * (double)qscale * (double)ksh[kt] * a->scale;
      };
      // 16-bit score: fp64 dot product of the 16-bit input values.
      auto score16 = [&](int r, long j) -> double {
        const float* x = qh + (size_t)(r0 + r) * D;
        const float* y = kh + (size_t)j * D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += (double)x[d] * (double)y[d];
        return acc * a->scale;
      };

      // Live key tiles of this query tile: some row of the tile sees some key of the tile.
      std::vector<long> lo(rows_in_tile), hi(rows_in_tile);
      for (int r = 0; r < rows_in_tile; ++r) g.visible(r0 + r, &lo[r], &hi[r]);
      auto tile_live = [&](int kt) {
        long c0 = (long)kt * g.bn, c1 = std::min<long>(g.Lk, c0 + g.bn) - 1;
        for (int r = 0; r < rows_in_tile; ++r)
          if (lo[r] <= hi[r] && lo[r] <= c1 && hi[r] >= c0) return true;
        return false;
      };

      // Routing of every key tile of this query tile.
      for (int kt = 0; kt < nkt; ++kt) tile_route[kt] = 0;
      if (!a->adaptive) {
        const uint64_t* mrow =
            a->mask ? a->mask + (((size_t)b * g.H + h) * nqt + qt) * a->mask_words : nullptr;
        for (int kt = 0; kt < nkt; ++kt) {
          if (!tile_live(kt)) continue;
          int gi = kt / a->group_tiles;
          int bit = mrow ? (int)((mrow[gi >> 6] >> (gi & 63)) & 1ull) : 1;
          tile_route[kt] = bit ? 1 : 2;
        }
      } else {
        // Look-ahead rule, ascending key tiles: t_r = 8-bit max of row r over its visible
        // keys in the tile; m_r = running max of the scores used so far (before this tile);
        // the tile is recomputed in 16 bits iff some row has t_r >= m_r - tau.
        for (int r = 0; r < rows_in_tile; ++r) m_run[r] = NEG_INF;
        const uint8_t* hint =
            a->route_hint ? a->route_hint + (((size_t)b * g.H + h) * nqt + qt) * nkt : nullptr;
        std::vector<double> t(rows_in_tile);
        for (int kt = 0; kt < nkt; ++kt) {
          if (!tile_live(kt)) continue;
          long c0 = (long)kt * g.bn, c1 = std::min<long>(g.Lk, c0 + g.bn) - 1;
          size_t ti = (((size_t)b * g.H + h) * nqt + qt) * nkt + kt;
          // Threshold skip (LATTE page: low-precision dot products filter the keys far below
          // the row maximum; here per tile): the tile is dropped iff every row with a visible
          // key in it has a running max and t_r < m_r - skip_tau.  Its margin: the smallest
          // (m_r - skip_tau) - t_r when dropped, else the largest t_r - (m_r - skip_tau).
          if (a->skip_tau != INF) {
            bool keep = false;
            double drop_margin = INF, keep_margin = NEG_INF;
            for (int r = 0; r < rows_in_tile; ++r) {
              long jl = std::max(lo[r], c0), jh = std::min(hi[r], c1);
              if (jl > jh) continue;
              double tr = NEG_INF;
              for (long j = jl; j <= jh; ++j) tr = std::max(tr, score8(r, j));
              double thr = m_run[r] - a->skip_tau;
              if (m_run[r] == NEG_INF || tr >= thr) {
                keep = true;
                keep_margin = std::max(keep_margin, m_run[r] == NEG_INF ? INF : tr - thr);
              } else {
                drop_margin = std::min(drop_margin, thr - tr);
              }
            }
            double sm = keep ? keep_margin : drop_margin;
            if (hint && sm < a->hint_margin && (hint[kt] == 1 || hint[kt] == 3 || hint[kt] == 4)) {
              const bool own = keep;
              keep = (hint[kt] != 4);
              if (a->hinted && keep != own) a->hinted[ti] = 1;
            }
            if (!keep) {
              tile_route[kt] = 4;
              if (a->margin) a->margin[ti] = sm;
              continue;
            }
            if (a->margin) a->margin[ti] = sm;
          }
          // Decision and its margin: the distance the deciding quantity is from the
          // threshold.  Flagged: the largest t_r - (m_r - tau) over voting rows (infinite
          // when some voting row has no running max yet).  Not flagged: the smallest
          // (m_r - tau) - t_r.
          bool flagged = false;
          double pass_margin = NEG_INF, fail_margin = INF;
          for (int r = 0; r < rows_in_tile; ++r) {
            t[r] = NEG_INF;
            long jl = std::max(lo[r], c0), jh = std::min(hi[r], c1);
            if (jl > jh) continue;
            for (long j = jl; j <= jh; ++j) t[r] = std::max(t[r], score8(r, j));
            double thr = m_run[r] - a->tau;
            if (t[r] >= thr) {
              flagged = true;
              pass_margin = std::max(pass_margin, m_run[r] == NEG_INF ? INF : t[r] - thr);
            } else {
              fail_margin = std::min(fail_margin, thr - t[r]);
            }
          }
          double margin = flagged ? pass_margin : fail_margin;
          // Where the decision is within `hint_margin` of flipping, two correct
          // implementations may disagree; follow the supplied routing map there.
          if (hint && margin < a->hint_margin && (hint[kt] == 1 || hint[kt] == 3)) {
            const bool own = flagged;
            flagged = (hint[kt] == 3);
            if (a->hinted && flagged != own) a->hinted[ti] = 1;
          }
          tile_route[kt] = flagged ? 3 : 1;
          if (a->margin) a->margin[ti] = std::min(a->margin[ti], margin);
          for (int r = 0; r < rows_in_tile; ++r) {
            long jl = std::max(lo[r], c0), jh = std::min(hi[r], c1);
            if (jl > jh) continue;
            double mx = NEG_INF;
            if (flagged)
              for (long j = jl; j <= jh; ++j) mx = std::max(mx, score16(r, j));
            else
              mx = t[r];
            m_run[r] = std::max(m_run[r], mx);
          }
        }
      }
      if (a->route)
        std::memcpy(a->route + (((size_t)b * g.H + h) * nqt + qt) * nkt, tile_route.data(), nkt);

      // Outputs of the requested rows: two-pass fp64 softmax over the routed scores.
      for (int s = I.r_begin; s < I.r_end; ++s) {
        int i = a->rows ? (int)a->rows[((size_t)b * g.H + h) * R + s] : s;
        int r = i - r0;
        double* orow = a->o + (((size_t)b * g.H + h) * R + s) * D;
        double* lrow = a->lse + ((size_t)b * g.H + h) * R + s;
        long jl = lo[r], jh = hi[r];
        if (jl > jh) {
          for (int d = 0; d < D; ++d) orow[d] = 0.0;
          *lrow = NEG_INF;
          continue;
        }
        double M = NEG_INF;
        for (long j = jl; j <= jh; ++j) {
          int rt = tile_route[j / g.bn];
          double sc = (rt == 4) ? NEG_INF : (rt == 1) ? score8(r, j) : score16(r, j);
          srow[j] = sc;
          M = std::max(M, sc);
        }
        double l = 0.0;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        for (long j = jl; j <= jh; ++j) {
          if (srow[j] == NEG_INF) continue;  // a dropped tile's keys
          double p = std::exp(srow[j] - M);
          l += p;
          const float* vj = vh + (size_t)j * D;
          for (int d = 0; d < D; ++d) orow[d] += p * (double)vj[d];
        }
        for (int d = 0; d < D; ++d) orow[d] /= l;
        *lrow = M + std::log(l);
        if (a->pv8) {
          // 8-bit exponentials against the running max, ascending key tiles, and an 8-bit P.V
          const size_t plane = (size_t)b * g.Hkv + kvh;
          const uint8_t* vct = vc.data() + plane * D * g.Lk;
          const float* vsc = vs.data() + plane * D;
          double m = NEG_INF, l8 = 0.0, mind = INF;
          for (int d = 0; d < D; ++d) orow[d] = 0.0;
          for (long kt = jl / g.bn; kt <= jh / g.bn; ++kt) {
            const long c0 = std::max(jl, kt * g.bn), c1 = std::min(jh, kt * g.bn + g.bn - 1);
            double tmax = NEG_INF;
            for (long j = c0; j <= c1; ++j) tmax = std::max(tmax, srow[j]);
            if (tmax == NEG_INF) continue;
            if (tmax > m) {
              if (m != NEG_INF) {
                const double f = std::exp(m - tmax);
                l8 *= f;
                for (int d = 0; d < D; ++d) orow[d] *= f;
              }
              m = tmax;
            }
            for (long j = c0; j <= c1; ++j) {
              if (srow[j] == NEG_INF) continue;
              double md;
              const double p8 = e4m3_round_pos(std::exp(srow[j] - m) * 256.0, &md);
              mind = std::min(mind, md);
              l8 += p8;
              for (int d = 0; d < D; ++d) orow[d] += p8 * e4m3_decode(vct[(size_t)d * g.Lk + j]);
            }
          }
          for (int d = 0; d < D; ++d) orow[d] = (double)vsc[d] * orow[d] / l8;
          if (a->pv8_margin) a->pv8_margin[((size_t)b * g.H + h) * R + s] = mind;
        }
      }
    }
  };
  int nt = a->threads > 0 ? a->threads : (int)std::thread::hardware_concurrency();
  if (nt < 1) nt = 1;
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  return 0;
}

}  // extern "C"
