// Per-block 8-bit quantiser (memory-bound) and routing-mask builder.
//
// Quantiser: TileMix page, section 2 "The Dual-Path Engine", item 2 (queries and keys are
// quantised to INT8 with per-block scale factors); LampAttention abstract (8-bit formats,
// here FP8 E4M3 as the option).  One CTA quantises one block of `blk` consecutive rows of one
// (batch, head), all D channels: a = max|x|, scale = a/127 (INT8) or a/448 (E4M3) as an IEEE
// fp32 quotient, code = round-to-nearest-even(x / scale) with an IEEE fp32 quotient, clamped
// to [-127, 127] or saturated to +-448.  The block is one contiguous run of rows*D 16-bit
// elements, read once with 16-byte vector loads kept in registers and written once with
// 8-byte vector stores: 2 bytes in, 1 byte out per element.
//
// Mask builder: TileMix page, section 2 "Packed Bitmasks" (one bit per group of adjacent key
// tiles, 0 = FP16, 1 = INT8).  The template is a seeded Bernoulli draw per group bit from a
// counter-based SplitMix64 hash (Steele, Lea, Flood 2014).
#pragma once

#include <cstdint>

namespace lamp {

constexpr int QUANT_THREADS = 256;
constexpr int QUANT_MAX_VEC = 16;  // 16-byte vectors per thread: 256*16*8 = 32768 elements

__device__ __forceinline__ float h16_to_f32(uint32_t bits, bool bf16) {
  if (bf16) return __uint_as_float(bits << 16);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool BF16, bool E4M3>
__global__ void __launch_bounds__(QUANT_THREADS) quant_kernel(const uint16_t* __restrict__ x,
                                                              uint8_t* __restrict__ codes,
                                                              float* __restrict__ scales, int L,
                                                              int D, int blk, int nb) {
  __shared__ float red[QUANT_THREADS / 32];
  const int blk_id = blockIdx.x;  // = outer * nb + block
  const int o = blk_id / nb, bi = blk_id - o * nb;
  const int r0 = bi * blk;
  const int rows = min(blk, L - r0);
  const size_t base = (static_cast<size_t>(o) * L + r0) * D;
  const int nvec = rows * D / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x + base);

  uint4 buf[QUANT_MAX_VEC];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < QUANT_MAX_VEC; ++k) {
    const int v = threadIdx.x + k * QUANT_THREADS;
    if (v < nvec) {
      buf[k] = __ldg(xv + v);
      const uint32_t w[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        amax = fmaxf(amax, fabsf(h16_to_f32(w[e] & 0xFFFFu, BF16)));
        amax = fmaxf(amax, fabsf(h16_to_f32(w[e] >> 16, BF16)));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int k = 1; k < QUANT_THREADS / 32; ++k) amax = fmaxf(amax, red[k]);

  const float s = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, E4M3 ? 448.0f : 127.0f);
  if (threadIdx.x == 0) scales[blk_id] = s;

  uint2* cv = reinterpret_cast<uint2*>(codes + base);
#pragma unroll
  for (int k = 0; k < QUANT_MAX_VEC; ++k) {
    const int v = threadIdx.x + k * QUANT_THREADS;
    if (v < nvec) {
      const uint32_t w[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
      uint32_t out[2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = h16_to_f32(w[e] & 0xFFFFu, BF16);
        const float x1 = h16_to_f32(w[e] >> 16, BF16);
        uint32_t pair;
        if (s == 0.0f) {
          pair = 0;
        } else if (E4M3) {
          pair = e4m3x2(__fdiv_rn(x0, s), __fdiv_rn(x1, s));
        } else {
          int c0 = __float2int_rn(__fdiv_rn(x0, s));
          int c1 = __float2int_rn(__fdiv_rn(x1, s));
          c0 = max(-127, min(127, c0));
          c1 = max(-127, min(127, c1));
          pair = (static_cast<uint32_t>(c0) & 0xFFu) | ((static_cast<uint32_t>(c1) & 0xFFu) << 8);
        }
        if (e & 1)
          out[e >> 1] |= pair << 16;
        else
          out[e >> 1] = pair;
      }
      cv[v] = make_uint2(out[0], out[1]);
    }
  }
}

// SplitMix64 step from state x: add the golden gamma, then the variant-13 finaliser.
__device__ __forceinline__ uint64_t splitmix64_step(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// One thread per mask word: rows = B*H*nQT mask rows of W words each.
__global__ void mask_kernel(uint64_t* __restrict__ mask, long long rows, int ng, int W,
                            double p_fp16, uint64_t seed) {
  const long long total = rows * W;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / W;
    const int w = static_cast<int>(i - row * W);
    uint64_t word = 0;
    for (int bit = 0; bit < 64; ++bit) {
      const int g = w * 64 + bit;
      if (g >= ng) break;
      const uint64_t idx = static_cast<uint64_t>(row) * static_cast<uint64_t>(ng) + g;
      const uint64_t u = splitmix64_step(seed ^ (idx * 0x9E3779B97F4A7C15ull));
      const double r = static_cast<double>(u >> 11) * 0x1.0p-53;
      if (!(r < p_fp16)) word |= 1ull << bit;
    }
    mask[i] = word;
  }
}

}  // namespace lamp
