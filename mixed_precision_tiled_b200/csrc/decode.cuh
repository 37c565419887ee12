// Decode with an 8-bit key/value cache (TileMix page, section 4: INT8 key/value caches for the
// decode phase, grouped-query attention).  One new query row per (batch, head) attends to the
// cached keys of its sequence; the cache holds 8-bit codes with per-block scales (blocks of BN
// rows, as the quantiser writes them for K).  Routing per key group from the packed mask:
//   8-bit route:  s = (q8 . k8) * sq * sk * scale   (exact int32 dot for INT8),
//   16-bit route: s = (q . k8) * sk * scale          (the full-precision query against the
//                                                     dequantised key: no 16-bit key is cached),
// values v = v8 * sv, softmax and P.V in fp32.
//
// The work is memory-bound (one pass over the cache), so it runs on the CUDA cores.  CTA
// (split, b * Hkv + kvh) serves all G query heads of one KV head from one read of its cache and
// walks a run of DEC_SPLIT_CHUNKS chunks of DEC_CHUNK keys: the chunks stream through a ring of
// shared-memory stages filled by bulk asynchronous copies (one thread issues them, an mbarrier
// per stage counts the bytes), so the next chunks' loads overlap the current chunk's
// arithmetic.  An online softmax per head runs across the CTA's chunks; the CTA writes one
// partial (m, l, O) per head and a second kernel merges the partials of each (b, h).
// Per chunk: scores with one thread per key (the key row read from shared memory in a rotated
// 16-byte order, free of bank conflicts), the chunk's softmax update with one warp per head, and
// P.V with the warps over keys and the lanes over channels, so that each value code is
// converted once for all heads of the group.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "ptx.cuh"

namespace lamp {

// threads of the split kernel: 8 warps, 16 at D = 256 (whose CTA is alone on its SM)
__host__ __device__ constexpr int dec_threads(int D) { return D == 256 ? 512 : 256; }
constexpr int DEC_CHUNK = 128;        // keys per pipeline stage
constexpr int DEC_STAGES = 2;         // stages of the shared-memory ring
constexpr int DEC_SPLIT_CHUNKS = 8;   // chunks per CTA (the split of the cache)
constexpr int DEC_MAX_G = 8;          // query heads per KV head

struct DecodeParams {
  const uint16_t* q;      // [B][H][D] 16-bit
  const uint8_t* q8;      // [B][H][D] codes
  const float* q_scale;   // [B][H]
  const uint8_t* k8;      // [B][Hkv][max_k][D]
  const float* k_scale;   // [B][Hkv][nKT]
  const uint8_t* v8;      // [B][Hkv][max_k][D]
  const float* v_scale;   // [B][Hkv][nKT]
  const int* len_k;       // [B] cached keys per sequence, or null (max_k)
  const uint64_t* mask;   // [B][H][1][W] or null (every group 8-bit)
  float* part;            // [B*H][nsplit][2 + D]: m, l, O (unnormalised)
  float* o;               // [B][H][D]
  float* lse;             // [B][H]
  int B, H, Hkv, G, max_k, nkt, bn, nsplit, mask_words, group_tiles;
  float scale;            // natural-log units
  int e4m3, bf16;
  uint32_t wait_us;       // limit of one bounded wait
};

__device__ __forceinline__ float dec_h16(uint16_t bits, bool bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(bits) << 16)
              : __half2float(__ushort_as_half(bits));
}

// E4M3 (OCP e4m3fn) code -> value: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
// holds the subnormals m/8 * 2^-6.  (Code 0x7F / 0xFF, NaN, is not produced by the quantiser.)
__device__ __forceinline__ float dec_e4m3(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  const float mag = (e == 0) ? static_cast<float>(m) * 0.001953125f  // m/8 * 2^-6
                             : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80u) ? -mag : mag;
}

// Two codes (bits 0-7 and 8-15 of c) -> two floats: E4M3 through the hardware conversion to a
// half pair (exact: every E4M3 value is an fp16 value), INT8 by sign-extending conversions.
template <bool E4M3>
__device__ __forceinline__ float2 dec_pair(uint32_t c) {
  if (E4M3) {
    uint32_t h2;
    asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h2) : "r"(c & 0xFFFFu));
    return __half22float2(*reinterpret_cast<__half2*>(&h2));
  }
  return make_float2(static_cast<float>(static_cast<int8_t>(c & 0xFFu)),
                     static_cast<float>(static_cast<int8_t>((c >> 8) & 0xFFu)));
}

template <bool E4M3>
__device__ __forceinline__ float dec_code(uint32_t c) {
  return E4M3 ? dec_e4m3(c) : static_cast<float>(static_cast<int8_t>(c));
}

// Shared-memory plan of the split kernel (bytes): the ring of key and value stages, then the
// query of every head (codes and values), scores, the scaled probabilities and the stage
// barriers.  At the end of the split the ring holds the cross-warp reduction of O.
template <int D>
struct DecSmem {
  static constexpr int STAGE = DEC_CHUNK * D;                         // one chunk of codes
  static constexpr int OFF_K = 0;                                     // + stage * STAGE
  static constexpr int OFF_V = DEC_STAGES * STAGE;                    // + stage * STAGE
  static constexpr int OFF_Q8 = 2 * DEC_STAGES * STAGE;               // [G][D] codes
  static constexpr int OFF_QF = OFF_Q8 + DEC_MAX_G * D;               // [G][D] fp32
  static constexpr int OFF_QE = OFF_QF + DEC_MAX_G * D * 4;           // [G][D] decoded E4M3 codes
  static constexpr int OFF_S = OFF_QE + DEC_MAX_G * D * 4;            // [G][CHUNK] fp32
  static constexpr int OFF_P = OFF_S + DEC_MAX_G * DEC_CHUNK * 4;     // [G][CHUNK] (p, p) pairs
  static constexpr int OFF_A = OFF_P + DEC_CHUNK * DEC_MAX_G * 8;     // [G] rescale factors
  static constexpr int OFF_ML = OFF_A + DEC_MAX_G * 4;                // [G][2] running m, l
  static constexpr int OFF_BAR = (OFF_ML + DEC_MAX_G * 8 + 7) & ~7;   // [STAGES] mbarriers
  static constexpr int BYTES = OFF_BAR + DEC_STAGES * 8;
  static_assert((dec_threads(D) / 32) * DEC_MAX_G * D * 4 <= 2 * DEC_STAGES * STAGE,
                "O reduction fits the ring");
  static_assert(STAGE % 16 == 0 && OFF_Q8 % 16 == 0 && OFF_QF % 16 == 0, "alignment");
};

// GM: the group size rounded up to a power of two (1, 2, 4 or 8), the compile-time bound of
// every per-head loop (the heads past G are skipped at run time)
template <int D, bool E4M3, int GM>
__global__ void __launch_bounds__(dec_threads(D)) decode_split_kernel(const DecodeParams p) {
  static_assert(D == 64 || D == 128 || D == 256, "head dimension");
  static_assert(GM == 1 || GM == 2 || GM == 4 || GM == 8, "group bound");
  constexpr int NT = dec_threads(D);
  constexpr int NHG = NT / DEC_CHUNK;           // head groups of the score phase
  constexpr int GH = (GM + NHG - 1) / NHG;      // heads per thread in the score phase
  using S = DecSmem<D>;
  constexpr int NW = NT / 32;
  constexpr int CPL = D / 32;            // channels per lane in the P.V phase
  constexpr int KPW = DEC_CHUNK / NW;    // keys per warp in the P.V phase
  constexpr int CPR = D / 16;            // 16-byte pieces per code row
  extern __shared__ __align__(16) uint8_t dsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + S::OFF_BAR);
  float* sc = reinterpret_cast<float*>(dsm + S::OFF_S);
  float2* pw = reinterpret_cast<float2*>(dsm + S::OFF_P);
  float* al = reinterpret_cast<float*>(dsm + S::OFF_A);
  float* ml = reinterpret_cast<float*>(dsm + S::OFF_ML);
  const float* qf = reinterpret_cast<const float*>(dsm + S::OFF_QF);
  const float* qe = reinterpret_cast<const float*>(dsm + S::OFF_QE);
  const uint32_t* q8w = reinterpret_cast<const uint32_t*>(dsm + S::OFF_Q8);

  const int G = p.G;
  const int split = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int len = p.len_k ? min(max(__ldg(p.len_k + b), 0), p.max_k) : p.max_k;
  const int nchunk = (len + DEC_CHUNK - 1) / DEC_CHUNK;
  const int cbeg = split * DEC_SPLIT_CHUNKS;
  const int cend = min(nchunk, cbeg + DEC_SPLIT_CHUNKS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool bf16 = p.bf16 != 0;
  const size_t row0 = static_cast<size_t>(bkv) * p.max_k;  // first cache row of this KV head
  const float NEG_INF = -__int_as_float(0x7f800000);
  const WaitCtx wc{0u, p.wait_us};

  // stage s holds chunk cbeg + s + k * STAGES; thread 0 issues the copies
  auto issue = [&](int c) {
    const int st = (c - cbeg) % DEC_STAGES;
    const int c0 = c * DEC_CHUNK;
    const uint32_t rows = static_cast<uint32_t>(min(DEC_CHUNK, p.max_k - c0));
    const uint32_t bytes = rows * D;
    mbar_arrive_expect_tx(&full[st], 2u * bytes);
    bulk_load(smem_u32(dsm + S::OFF_K + st * S::STAGE), p.k8 + (row0 + c0) * D, bytes, &full[st]);
    bulk_load(smem_u32(dsm + S::OFF_V + st * S::STAGE), p.v8 + (row0 + c0) * D, bytes, &full[st]);
  };
  if (tid == 0) {
    for (int s = 0; s < DEC_STAGES; ++s) mbar_init(&full[s], 1);
    fence_mbarrier_init();
    for (int c = cbeg; c < min(cend, cbeg + DEC_STAGES); ++c) issue(c);
  }
  // the G query rows of this KV group: values and codes; running max and sum per head
  for (int i = tid; i < G * D; i += NT) {
    const int g = i / D, d = i - g * D;
    const size_t qi = static_cast<size_t>(b * p.H + kvh * G + g) * D + d;
    reinterpret_cast<float*>(dsm + S::OFF_QF)[g * D + d] = dec_h16(p.q[qi], bf16);
  }
  for (int i = tid; i < G * D / 4; i += NT) {
    const int g = i / (D / 4), w = i - g * (D / 4);
    const uint32_t word = __ldg(
        reinterpret_cast<const uint32_t*>(p.q8 + static_cast<size_t>(b * p.H + kvh * G + g) * D) + w);
    reinterpret_cast<uint32_t*>(dsm + S::OFF_Q8)[g * (D / 4) + w] = word;
    if (E4M3) {
      float* qd = reinterpret_cast<float*>(dsm + S::OFF_QE) + g * D + 4 * w;
      const float2 a = dec_pair<true>(word), c = dec_pair<true>(word >> 16);
      qd[0] = a.x; qd[1] = a.y; qd[2] = c.x; qd[3] = c.y;
    }
  }
  if (tid < G) {
    ml[2 * tid] = NEG_INF;
    ml[2 * tid + 1] = 0.0f;
  }
  // the scores of this thread's key: heads g = hh, hh + NHG, ... (hh = tid / 128)
  const int hh = tid / DEC_CHUNK, jl = tid - hh * DEC_CHUNK;
  float sqh[GH];
#pragma unroll
  for (int k = 0; k < GH; ++k) {
    const int g = hh + NHG * k;
    sqh[k] = (g < G) ? __ldg(p.q_scale + b * p.H + kvh * G + g) : 0.0f;
  }
  uint64_t acc[GM][CPL / 2];  // O accumulators of this lane's channels, as f32x2 pairs
#pragma unroll
  for (int g = 0; g < GM; ++g)
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) acc[g][e] = 0ull;
  __syncthreads();

  bool ok = true;
  for (int c = cbeg; c < cend; ++c) {
    const int st = (c - cbeg) % DEC_STAGES;
    const uint32_t par = static_cast<uint32_t>((c - cbeg) / DEC_STAGES) & 1u;
    const int c0 = c * DEC_CHUNK;
    const int rows = min(DEC_CHUNK, len - c0);  // keys of this chunk in the sequence
    if (!mbar_wait(&full[st], par, wc, W_FULL)) ok = false;
    const uint8_t* ksm = dsm + S::OFF_K + st * S::STAGE;
    const uint8_t* vsm = dsm + S::OFF_V + st * S::STAGE;

    // ---- scores
    {
      const int j = c0 + jl;
      const bool live = ok && jl < rows;
      const int kt = j / p.bn;
      const float sk = live ? __ldg(p.k_scale + static_cast<size_t>(bkv) * p.nkt + kt) : 0.0f;
      const int gi = kt / p.group_tiles;
      // routing word of each of this thread's heads (loaded ahead of the dot products)
      uint64_t mw[GH];
#pragma unroll
      for (int k = 0; k < GH; ++k) {
        const int g = hh + NHG * k;
        mw[k] = ~0ull;
        if (live && p.mask && g < G)
          mw[k] = __ldg(reinterpret_cast<const unsigned long long*>(p.mask) +
                        static_cast<size_t>(b * p.H + kvh * G + g) * p.mask_words + (gi >> 6));
      }
      // heads scored from the INT8 codes (dp4a) and heads scored in floats: the 16-bit route
      // (full-precision query, dequantised key) and the E4M3 8-bit route (decoded codes)
      bool eight[GH];
      bool any_float = false;
#pragma unroll
      for (int k = 0; k < GH; ++k) {
        eight[k] = ((mw[k] >> (gi & 63)) & 1ull) != 0;
        any_float = any_float || ((hh + NHG * k) < G && (E4M3 || !eight[k]));
      }
      int ia[GH];
      uint64_t fa[GH];  // float-path dot products as f32x2 partial sums (even, odd channels)
#pragma unroll
      for (int k = 0; k < GH; ++k) {
        ia[k] = 0;
        fa[k] = 0ull;
      }
      if (live) {
        // the key row's 16-byte pieces are read in a rotated order (piece (i + jl) % CPR at step
        // i) so that a warp's lanes hit distinct banks, and the query at the matching channels
        const uint4* krow = reinterpret_cast<const uint4*>(ksm + jl * D);
        // float heads (16-bit route, E4M3 codes): piece i converted once for all of them
        auto float_piece = [&](int i, const uint4& kq) {
          const int ci = (i + jl) & (CPR - 1);
          uint64_t kf[8];  // the piece's 16 codes as f32x2 pairs
          const uint32_t ka[4] = {kq.x, kq.y, kq.z, kq.w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float2 f0 = dec_pair<E4M3>(ka[w]), f1 = dec_pair<E4M3>(ka[w] >> 16);
            kf[2 * w] = f2_pack(f0.x, f0.y);
            kf[2 * w + 1] = f2_pack(f1.x, f1.y);
          }
#pragma unroll
          for (int k = 0; k < GH; ++k) {
            const int g = hh + NHG * k;
            if (g >= G) break;
            if (!E4M3 && eight[k]) continue;
            const ulonglong2* q4 =
                reinterpret_cast<const ulonglong2*>((eight[k] ? qe : qf) + g * D + 16 * ci);
            uint64_t f = fa[k];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const ulonglong2 qq = q4[w];
              f = f2_fma(qq.x, kf[2 * w], f);
              f = f2_fma(qq.y, kf[2 * w + 1], f);
            }
            fa[k] = f;
          }
        };
        // INT8 heads: four dp4a per piece
        auto int_piece = [&](int i, const uint4& kq, int k, int g) {
          const uint4 qq = reinterpret_cast<const uint4*>(q8w + g * (D / 4))[(i + jl) & (CPR - 1)];
          ia[k] = __dp4a(static_cast<int>(qq.x), static_cast<int>(kq.x), ia[k]);
          ia[k] = __dp4a(static_cast<int>(qq.y), static_cast<int>(kq.y), ia[k]);
          ia[k] = __dp4a(static_cast<int>(qq.z), static_cast<int>(kq.z), ia[k]);
          ia[k] = __dp4a(static_cast<int>(qq.w), static_cast<int>(kq.w), ia[k]);
        };
        if constexpr (D <= 128) {
          // the whole row in registers; the dp4a chains of each head fully unrolled
          uint4 kr[CPR];
#pragma unroll
          for (int i = 0; i < CPR; ++i) kr[i] = krow[(i + jl) & (CPR - 1)];
          if (!E4M3) {
#pragma unroll
            for (int k = 0; k < GH; ++k) {
              const int g = hh + NHG * k;
              if (g >= G) break;
              if (!eight[k]) continue;
#pragma unroll
              for (int i = 0; i < CPR; ++i) int_piece(i, kr[i], k, g);
            }
          }
          if (any_float) {
#pragma unroll
            for (int i = 0; i < CPR; ++i) float_piece(i, kr[i]);
          }
        } else {
          // D = 256: piece by piece (the row would not fit the register budget of 512 threads)
#pragma unroll 2
          for (int i = 0; i < CPR; ++i) {
            const uint4 kq = krow[(i + jl) & (CPR - 1)];
            if (!E4M3) {
#pragma unroll
              for (int k = 0; k < GH; ++k) {
                const int g = hh + NHG * k;
                if (g >= G) break;
                if (eight[k]) int_piece(i, kq, k, g);
              }
            }
            if (any_float) float_piece(i, kq);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < GH; ++k) {
        const int g = hh + NHG * k;
        if (g >= G) break;
        float s = NEG_INF;
        if (live) {
          float f0, f1;
          f2_unpack(fa[k], f0, f1);
          if (eight[k])
            s = (E4M3 ? f0 + f1 : static_cast<float>(ia[k])) * sqh[k] * sk * p.scale;
          else
            s = (f0 + f1) * sk * p.scale;
        }
        sc[g * DEC_CHUNK + jl] = s;
      }
    }
    __syncthreads();

    // ---- softmax update, warp g for head g: chunk max, rescale factor, p * v_scale
    if (warp < G) {
      const int g = warp;
      // value scales of the chunk's key blocks (a chunk spans one block of 128 keys or two of
      // 64), read before the reduction so that their latency overlaps it
      const int kt0 = c0 / p.bn;
      const float vs0 = __ldg(p.v_scale + static_cast<size_t>(bkv) * p.nkt + kt0);
      const float vs1 = (p.bn < DEC_CHUNK && kt0 + 1 < p.nkt)
                            ? __ldg(p.v_scale + static_cast<size_t>(bkv) * p.nkt + kt0 + 1) : 0.0f;
      float m = ml[2 * g], l = ml[2 * g + 1];
      float sv[DEC_CHUNK / 32];
      float cm = NEG_INF;
#pragma unroll
      for (int k = 0; k < DEC_CHUNK / 32; ++k) {
        sv[k] = sc[g * DEC_CHUNK + k * 32 + lane];
        cm = fmaxf(cm, sv[k]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xFFFFFFFFu, cm, o));
      const float mn = fmaxf(m, cm);
      const float a = (m == NEG_INF) ? 0.0f : __expf(m - mn);
      float ls = 0.0f;
#pragma unroll
      for (int k = 0; k < DEC_CHUNK / 32; ++k) {
        const int jj = k * 32 + lane;
        const float pr = (sv[k] == NEG_INF) ? 0.0f : __expf(sv[k] - mn);
        ls += pr;
        const float pv = pr * ((jj < p.bn) ? vs0 : vs1);
        pw[g * DEC_CHUNK + jj] = make_float2(pv, pv);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o);
      if (lane == 0) {
        al[g] = a;
        ml[2 * g] = mn;
        ml[2 * g + 1] = l * a + ls;
      }
    }
    __syncthreads();

    // ---- P.V: warp w takes keys w * KPW .. + KPW of the chunk, lane l channels l * CPL ..
    // (f32x2 FMAs: each weight is stored as a (p, p) pair, the channels go in pairs)
    {
#pragma unroll
      for (int g = 0; g < GM; ++g) {
        if (g >= G) break;
        const uint64_t a2 = f2_pack(al[g], al[g]);
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) acc[g][e] = f2_fma(acc[g][e], a2, 0ull);
      }
      const int jb = warp * KPW, je = min(jb + KPW, rows);
      for (int jj = jb; jj < je; ++jj) {
        const uint8_t* vrow = vsm + jj * D + lane * CPL;
        uint32_t vw[(CPL + 3) / 4];
        if (CPL == 8) {
          const uint2 t = *reinterpret_cast<const uint2*>(vrow);
          vw[0] = t.x;
          vw[1] = t.y;
        } else if (CPL == 4) {
          vw[0] = *reinterpret_cast<const uint32_t*>(vrow);
        } else {
          vw[0] = *reinterpret_cast<const uint16_t*>(vrow);
        }
        uint64_t vv[CPL / 2];
#pragma unroll
        for (int e = 0; e < CPL; e += 2) {
          const float2 f = dec_pair<E4M3>(vw[e >> 2] >> (8 * (e & 3)));
          vv[e / 2] = f2_pack(f.x, f.y);
        }
        const uint64_t* pcol = reinterpret_cast<const uint64_t*>(pw + jj);
#pragma unroll
        for (int g = 0; g < GM; ++g) {
          if (g >= G) break;
          const uint64_t pg = pcol[g * DEC_CHUNK];  // (the whole warp reads one address)
#pragma unroll
          for (int e = 0; e < CPL / 2; ++e) acc[g][e] = f2_fma(pg, vv[e], acc[g][e]);
        }
      }
    }
    __syncthreads();  // every thread is done with this stage and with the scores / weights
    if (tid == 0 && c + DEC_STAGES < cend) issue(c + DEC_STAGES);
  }

  // ---- the partial of each head: m, l and O summed over the warps (in the ring's space)
  float* red = reinterpret_cast<float*>(dsm);  // [NW][G][D]
#pragma unroll
  for (int g = 0; g < GM; ++g) {
    if (g >= G) break;
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) {
      float lo, hi;
      f2_unpack(acc[g][e], lo, hi);
      red[(warp * DEC_MAX_G + g) * D + lane * CPL + 2 * e] = lo;
      red[(warp * DEC_MAX_G + g) * D + lane * CPL + 2 * e + 1] = hi;
    }
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += NT) {
    const int g = i / D, d = i - g * D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += red[(w * DEC_MAX_G + g) * D + d];
    const int h = kvh * G + g;
    float* out = p.part + (static_cast<size_t>(b * p.H + h) * p.nsplit + split) * (2 + D);
    out[2 + d] = s;
    if (d == 0) {
      out[0] = ml[2 * g];
      out[1] = ml[2 * g + 1];
    }
  }
}

// Merge the partials of one (b, h): M = max m_s, l = sum l_s e^(m_s - M), O = sum O_s e^(m_s - M) / l,
// lse = M + ln l.  A sequence with no cached key gets O = 0 and lse = -inf.  The split weights
// e^(m_s - M) are computed once, in parallel, into shared memory; every thread then sums its
// channel over the splits with independent, coalesced loads.
constexpr int DEC_COMBINE_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(DEC_COMBINE_THREADS) decode_combine_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) float wsm[];  // [nsplit] weights, then [32] reduction scratch
  float* scratch = wsm + p.nsplit;
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = DEC_COMBINE_THREADS / 32;
  const float* part = p.part + static_cast<size_t>(bh) * p.nsplit * (2 + D);
  const float NEG_INF = -__int_as_float(0x7f800000);
  float m = NEG_INF;
  for (int s = tid; s < p.nsplit; s += DEC_COMBINE_THREADS) m = fmaxf(m, part[s * (2 + D)]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) scratch[warp] = m;
  __syncthreads();
  float M = NEG_INF;
#pragma unroll
  for (int w = 0; w < NW; ++w) M = fmaxf(M, scratch[w]);
  float l = 0.0f;
  for (int s = tid; s < p.nsplit; s += DEC_COMBINE_THREADS) {
    const float ms = part[s * (2 + D)];
    const float wt = (ms == NEG_INF) ? 0.0f : __expf(ms - M);
    wsm[s] = wt;
    l += part[s * (2 + D) + 1] * wt;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
  __syncthreads();  // (scratch reused, weights complete)
  if (lane == 0) scratch[NW + warp] = l;
  __syncthreads();
  float L = 0.0f;
#pragma unroll
  for (int w = 0; w < NW; ++w) L += scratch[NW + w];
  const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
  for (int d = tid; d < D; d += DEC_COMBINE_THREADS) {
    float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
    int s = 0;
    for (; s + 4 <= p.nsplit; s += 4) {
      o0 = fmaf(part[(s + 0) * (2 + D) + 2 + d], wsm[s + 0], o0);
      o1 = fmaf(part[(s + 1) * (2 + D) + 2 + d], wsm[s + 1], o1);
      o2 = fmaf(part[(s + 2) * (2 + D) + 2 + d], wsm[s + 2], o2);
      o3 = fmaf(part[(s + 3) * (2 + D) + 2 + d], wsm[s + 3], o3);
    }
    for (; s < p.nsplit; ++s) o0 = fmaf(part[s * (2 + D) + 2 + d], wsm[s], o0);
    p.o[static_cast<size_t>(bh) * D + d] = ((o0 + o1) + (o2 + o3)) * inv;
  }
  if (tid == 0) p.lse[bh] = (L > 0.0f) ? M + logf(L) : NEG_INF;
}

}  // namespace lamp
