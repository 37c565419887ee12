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
// merges the partials of each (b, h).  The chunk's key and value rows are loaded cooperatively
// (coalesced) into XOR-swizzled shared memory; each thread then reads its own key row.
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

template <bool E4M3>
__device__ __forceinline__ float dec_code(uint32_t c) {
  return E4M3 ? dec_e4m3(c) : static_cast<float>(static_cast<int8_t>(c));
}

template <int D, bool E4M3>
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
  // [CHUNK][D] value codes; 16-byte chunk c of row j sits at chunk c ^ (j & SW): the row stores
  // of consecutive threads and the row reads of a warp are both free of bank conflicts
  uint8_t* vsm = reinterpret_cast<uint8_t*>(stat + 2 * DEC_MAX_G);
  uint8_t* ksm = vsm + DEC_CHUNK * D;  // [CHUNK][D] key codes, same swizzle
  constexpr int SW = (D / 16 >= 8) ? 7 : (D / 16 - 1);

  const int G = p.G;
  const int split = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int len = p.len_k ? min(max(__ldg(p.len_k + b), 0), p.max_k) : p.max_k;
  const int c0 = split * DEC_CHUNK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool bf16 = p.bf16 != 0;
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

  // scores: one key per thread, all heads of the group.  The key row stays in registers; the
  // head loop is not unrolled (the unrolled body of every head overflowed the instruction
  // cache).
  {
    const int j = c0 + tid;
    const bool live = j < len;
    const int kt = j / p.bn;
    const float sk = live ? __ldg(p.k_scale + static_cast<size_t>(bkv) * p.nkt + kt) : 0.0f;
    const int gi = kt / p.group_tiles;
    // the chunk's key and value rows, loaded cooperatively (a warp reads whole rows: coalesced)
    // into swizzled shared memory; each thread then reads its own key row from there
    {
      constexpr int CPR = D / 16;  // 16-byte chunks per row
      const int rows = min(DEC_CHUNK, len - c0);
      const uint4* kbase = reinterpret_cast<const uint4*>(p.k8 + (cache_row0 + c0) * D);
      const uint4* vbase = reinterpret_cast<const uint4*>(p.v8 + (cache_row0 + c0) * D);
      uint4 kt_[DEC_CHUNK * CPR / DEC_THREADS], vt_[DEC_CHUNK * CPR / DEC_THREADS];
#pragma unroll
      for (int u = 0; u < DEC_CHUNK * CPR / DEC_THREADS; ++u) {
        const int idx = u * DEC_THREADS + tid, r = idx / CPR;
        if (r < rows) {
          kt_[u] = __ldg(kbase + idx);
          vt_[u] = __ldg(vbase + idx);
        }
      }
#pragma unroll
      for (int u = 0; u < DEC_CHUNK * CPR / DEC_THREADS; ++u) {
        const int idx = u * DEC_THREADS + tid, r = idx / CPR, c = idx - r * CPR;
        if (r < rows) {
          reinterpret_cast<uint4*>(ksm + r * D)[c ^ (r & SW)] = kt_[u];
          reinterpret_cast<uint4*>(vsm + r * D)[c ^ (r & SW)] = vt_[u];
        }
      }
    }
    __syncthreads();
    uint32_t kw[D / 4];
    if (live) {
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        const uint4 kr = reinterpret_cast<const uint4*>(ksm + tid * D)[i ^ (tid & SW)];
        kw[4 * i] = kr.x;
        kw[4 * i + 1] = kr.y;
        kw[4 * i + 2] = kr.z;
        kw[4 * i + 3] = kr.w;
      }
    }
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
      float s = -__int_as_float(0x7f800000);
      if (live) {
        const int h = kvh * G + g;
        bool eight = true;
        if (p.mask) {
          const uint64_t w = __ldg(reinterpret_cast<const unsigned long long*>(p.mask) +
                                   static_cast<size_t>(b * p.H + h) * p.mask_words + (gi >> 6));
          eight = ((w >> (gi & 63)) & 1ull) != 0;
        }
        if (eight) {
          const uint32_t* qw = q8w + g * (D / 4);
          const float sq = __ldg(p.q_scale + b * p.H + h);
          if (!E4M3) {
            int acc = 0;
#pragma unroll
            for (int i = 0; i < D / 4; ++i) acc = __dp4a(static_cast<int>(qw[i]), static_cast<int>(kw[i]), acc);
            s = static_cast<float>(acc) * sq * sk * p.scale;
          } else {
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < D / 4; ++i)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                acc = fmaf(dec_e4m3((qw[i] >> (8 * e)) & 0xFFu), dec_e4m3((kw[i] >> (8 * e)) & 0xFFu), acc);
            s = acc * sq * sk * p.scale;
          }
        } else {
          const float* qv = qf + g * D;
          float acc = 0.0f;
#pragma unroll
          for (int i = 0; i < D / 4; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              acc = fmaf(qv[4 * i + e], dec_code<E4M3>((kw[i] >> (8 * e)) & 0xFFu), acc);
          s = acc * sk * p.scale;
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
  float vsc[DEC_CHUNK / 64];  // value scales of the chunk's key tiles (BN >= 64)
#pragma unroll
  for (int i = 0; i < DEC_CHUNK / 64; ++i) {
    const int kt = c0 / p.bn + i;
    vsc[i] = (kt < p.nkt) ? __ldg(p.v_scale + static_cast<size_t>(bkv) * p.nkt + kt) : 0.0f;
  }
  for (int jj = warp; jj < jend; jj += NW) {
    const int j = c0 + jj;
    // lane's DL bytes of row jj: logical chunk (lane * DL) / 16, stored at chunk ^ (jj & SW)
    const int lc = (lane * DL) >> 4;
    const uint8_t* vrow = vsm + jj * D + ((lc ^ (jj & SW)) << 4) + ((lane * DL) & 15);
    uint32_t vw[(DL + 3) / 4];
    if (DL == 8) {
      const uint2 t = *reinterpret_cast<const uint2*>(vrow);
      vw[0] = t.x;
      vw[1] = t.y;
    } else if (DL == 4) {
      vw[0] = *reinterpret_cast<const uint32_t*>(vrow);
    } else {
      vw[0] = *reinterpret_cast<const uint16_t*>(vrow);
    }
    const float sv = vsc[(j / p.bn) - c0 / p.bn];
    float vv[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) vv[e] = dec_code<E4M3>((vw[e >> 2] >> (8 * (e & 3))) & 0xFFu) * sv;
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
