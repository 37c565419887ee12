// Decode with an 8-bit key/value cache (TileMix page, section 4: INT8 key/value caches for the
// decode phase, grouped-query attention).  One new query row per (batch, head) attends to the
// cached keys of its sequence; the cache holds 8-bit codes with per-block scales (blocks of BN
// rows, as the quantiser writes them for K).  Routing per key group from the packed mask:
//   8-bit route:  s = (q8 . k8) * sq * sk * scale   (exact int32 dot for INT8),
//   16-bit route: s = (q . k8) * sk * scale          (the full-precision query against the
//                                                     dequantised key: no 16-bit key is cached),
// values v = v8 * sv, softmax and P.V in fp32.
//
// The work is memory-bound (one pass over the cache), so it runs on the CUDA cores with the
// cache split across CTAs: CTA (chunk, b * Hkv + kvh) reads CHUNK keys of one KV head once for
// all G query heads of its group, and writes a partial (m, l, O) per head; a second kernel
// merges the partials of each (b, h).  Loads are 16-byte (keys, one row per thread) and
// row-coalesced (values, a warp per key row).
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "ptx.cuh"

namespace lamp {

constexpr int DEC_THREADS = 256;
constexpr int DEC_CHUNK = 256;  // keys per CTA (one per thread in the score phase)
constexpr int DEC_MAX_G = 8;    // query heads per KV head

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

__device__ __forceinline__ float dec_code(uint32_t c, bool e4m3) {
  return e4m3 ? dec_e4m3(c) : static_cast<float>(static_cast<int8_t>(c));
}

template <int D>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_split_kernel(const DecodeParams p) {
  static_assert(D == 64 || D == 128 || D == 256, "head dimension");
  constexpr int NW = DEC_THREADS / 32;
  constexpr int DL = D / 32;  // channels per lane in the P.V phase
  extern __shared__ __align__(16) float dsm[];
  float* sc = dsm;                                    // [G][CHUNK] scores, then probabilities
  float* qf = sc + DEC_MAX_G * DEC_CHUNK;             // [G][D] query values
  uint32_t* q8w = reinterpret_cast<uint32_t*>(qf + DEC_MAX_G * D);  // [G][D/4] query codes
  float* red = reinterpret_cast<float*>(q8w + DEC_MAX_G * D / 4);   // [NW][G][D] P.V partials
  float* stat = red + NW * DEC_MAX_G * D;             // [G][2] chunk max and sum

  const int G = p.G;
  const int split = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int len = p.len_k ? min(max(__ldg(p.len_k + b), 0), p.max_k) : p.max_k;
  const int c0 = split * DEC_CHUNK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool e4m3 = p.e4m3 != 0, bf16 = p.bf16 != 0;
  const size_t cache_row0 = static_cast<size_t>(bkv) * p.max_k;  // first row of this KV head

  // the G query rows of this KV group: values and codes
  for (int i = tid; i < G * D; i += DEC_THREADS) {
    const int g = i / D, d = i - g * D;
    const size_t qi = static_cast<size_t>(b * p.H + kvh * G + g) * D + d;
    qf[g * D + d] = dec_h16(p.q[qi], bf16);
  }
  for (int i = tid; i < G * D / 4; i += DEC_THREADS) {
    const int g = i / (D / 4), w = i - g * (D / 4);
    q8w[g * (D / 4) + w] = __ldg(reinterpret_cast<const uint32_t*>(
        p.q8 + static_cast<size_t>(b * p.H + kvh * G + g) * D) + w);
  }
  __syncthreads();

  // scores: one key per thread, all heads of the group, 16 bytes of the key row at a time
  {
    const int j = c0 + tid;
    const bool live = j < len;
    const int kt = j / p.bn;
    const float sk = live ? __ldg(p.k_scale + static_cast<size_t>(bkv) * p.nkt + kt) : 0.0f;
    const int gi = kt / p.group_tiles;
    uint32_t eight = (1u << G) - 1u;  // bit g: head g takes the 8-bit route for this key
    if (p.mask && live) {
      for (int g = 0; g < G; ++g) {
        const uint64_t w = __ldg(reinterpret_cast<const unsigned long long*>(p.mask) +
                                 static_cast<size_t>(b * p.H + kvh * G + g) * p.mask_words +
                                 (gi >> 6));
        if (((w >> (gi & 63)) & 1ull) == 0) eight &= ~(1u << g);
      }
    }
    int acc8[DEC_MAX_G];
    float accf[DEC_MAX_G];
#pragma unroll
    for (int g = 0; g < DEC_MAX_G; ++g) {
      acc8[g] = 0;
      accf[g] = 0.0f;
    }
    if (live) {
      const uint4* src = reinterpret_cast<const uint4*>(p.k8 + (cache_row0 + j) * D);
#pragma unroll 2
      for (int i = 0; i < D / 16; ++i) {
        const uint4 kr = __ldg(src + i);
        const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
        for (int g = 0; g < DEC_MAX_G; ++g) {
          if (g >= G) break;
          if ((eight >> g) & 1u) {
            const uint32_t* qw = q8w + g * (D / 4) + 4 * i;
            if (!e4m3) {
#pragma unroll
              for (int w = 0; w < 4; ++w)
                acc8[g] = __dp4a(static_cast<int>(qw[w]), static_cast<int>(kw[w]), acc8[g]);
            } else {
#pragma unroll
              for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  accf[g] = fmaf(dec_e4m3((qw[w] >> (8 * e)) & 0xFFu),
                                 dec_e4m3((kw[w] >> (8 * e)) & 0xFFu), accf[g]);
            }
          } else {
            const float* qv = qf + g * D + 16 * i;
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                accf[g] = fmaf(qv[4 * w + e], dec_code((kw[w] >> (8 * e)) & 0xFFu, e4m3), accf[g]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < DEC_MAX_G; ++g) {
      if (g >= G) break;
      float s = -__int_as_float(0x7f800000);
      if (live) {
        if ((eight >> g) & 1u) {
          const float sq = __ldg(p.q_scale + b * p.H + kvh * G + g);
          s = (e4m3 ? accf[g] : static_cast<float>(acc8[g])) * sq * sk * p.scale;
        } else {
          s = accf[g] * sk * p.scale;
        }
      }
      sc[g * DEC_CHUNK + tid] = s;
    }
  }
  __syncthreads();

  // per head: chunk max, probabilities p = e^(s - m), their sum (warp g takes head g)
  for (int g = warp; g < G; g += NW) {
    float m = -__int_as_float(0x7f800000);
    for (int i = lane; i < DEC_CHUNK; i += 32) m = fmaxf(m, sc[g * DEC_CHUNK + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    float l = 0.0f;
    for (int i = lane; i < DEC_CHUNK; i += 32) {
      const float s = sc[g * DEC_CHUNK + i];
      const float pr = (s == -__int_as_float(0x7f800000)) ? 0.0f : __expf(s - m);
      sc[g * DEC_CHUNK + i] = pr;
      l += pr;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
    if (lane == 0) {
      stat[2 * g] = m;
      stat[2 * g + 1] = l;
    }
  }
  __syncthreads();

  // P.V: warp w takes keys w, w + NW, ...; lane l holds channels [l * DL, l * DL + DL)
  float acc[DEC_MAX_G][DL];
#pragma unroll
  for (int g = 0; g < DEC_MAX_G; ++g)
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[g][e] = 0.0f;
  const int jend = min(DEC_CHUNK, len - c0);
  for (int jj = warp; jj < jend; jj += NW) {
    const int j = c0 + jj;
    const uint8_t* vrow = p.v8 + (cache_row0 + j) * D + lane * DL;
    uint32_t vw[(DL + 3) / 4];
    if (DL == 8) {
      const uint2 t = __ldg(reinterpret_cast<const uint2*>(vrow));
      vw[0] = t.x;
      vw[1] = t.y;
    } else if (DL == 4) {
      vw[0] = __ldg(reinterpret_cast<const uint32_t*>(vrow));
    } else {
      vw[0] = __ldg(reinterpret_cast<const uint16_t*>(vrow));
    }
    const float sv = __ldg(p.v_scale + static_cast<size_t>(bkv) * p.nkt + j / p.bn);
    float vv[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) vv[e] = dec_code((vw[e >> 2] >> (8 * (e & 3))) & 0xFFu, e4m3) * sv;
#pragma unroll
    for (int g = 0; g < DEC_MAX_G; ++g) {
      if (g >= G) break;
      const float pr = sc[g * DEC_CHUNK + jj];
#pragma unroll
      for (int e = 0; e < DL; ++e) acc[g][e] = fmaf(pr, vv[e], acc[g][e]);
    }
  }
#pragma unroll
  for (int g = 0; g < DEC_MAX_G; ++g) {
    if (g >= G) break;
#pragma unroll
    for (int e = 0; e < DL; ++e) red[(warp * DEC_MAX_G + g) * D + lane * DL + e] = acc[g][e];
  }
  __syncthreads();

  // the partial of each head: m, l, O = sum over the warps
  for (int i = tid; i < G * D; i += DEC_THREADS) {
    const int g = i / D, d = i - g * D;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += red[(w * DEC_MAX_G + g) * D + d];
    const int h = kvh * G + g;
    float* out = p.part + (static_cast<size_t>(b * p.H + h) * p.nsplit + split) * (2 + D);
    out[2 + d] = s;
    if (d == 0) {
      out[0] = stat[2 * g];
      out[1] = stat[2 * g + 1];
    }
  }
}

// Merge the partials of one (b, h): M = max m_s, l = sum l_s e^(m_s - M), O = sum O_s e^(m_s - M) / l,
// lse = M + ln l.  A sequence with no cached key gets O = 0 and lse = -inf.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const float* part = p.part + static_cast<size_t>(bh) * p.nsplit * (2 + D);
  const float NEG_INF = -__int_as_float(0x7f800000);
  float M = NEG_INF;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, part[s * (2 + D)]);
  float l = 0.0f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float m = part[s * (2 + D)];
    if (m != NEG_INF) l += part[s * (2 + D) + 1] * __expf(m - M);
  }
  const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float o = 0.0f;
    for (int s = 0; s < p.nsplit; ++s) {
      const float m = part[s * (2 + D)];
      if (m != NEG_INF) o += part[s * (2 + D) + 2 + d] * __expf(m - M);
    }
    p.o[static_cast<size_t>(bh) * D + d] = o * inv;
  }
  if (threadIdx.x == 0) p.lse[bh] = (l > 0.0f) ? M + logf(l) : NEG_INF;
}

}  // namespace lamp
