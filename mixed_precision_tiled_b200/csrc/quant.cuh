// Per-block 8-bit quantiser (memory-bound) and routing-mask builder.
//
// Quantiser: TileMix page, section 2 "The Dual-Path Engine", item 2 (queries and keys are
// quantised to INT8 with per-block scale factors); LampAttention abstract (8-bit formats,
// here FP8 E4M3 as the option).  One CTA quantises one block of `blk` consecutive rows of one
// (batch, head), all D channels: a = max|x|, scale = a/127 (INT8) or a/448 (E4M3) as an IEEE
// fp32 quotient, code = round-to-nearest-even(x / scale) with an IEEE fp32 quotient, clamped
// to [-127, 127] or saturated to +-448.  The block is one contiguous run of rows*D 16-bit
// elements, read once with 16-byte vector loads kept in registers and written once with
// 8-byte vector stores: 2 bytes in, 1 byte out per element.  Q and K are quantised by one
// launch.
//
// Mask builders: TileMix page, section 2 "Packed Bitmasks" (one bit per group of adjacent key
// tiles, 0 = FP16, 1 = INT8).  Two templates: a seeded Bernoulli draw per group bit from a
// counter-based SplitMix64 hash (Steele, Lea, Flood 2014), and a structured static template
// (sink, local band and strided groups in 16 bits; section 4 "static, data-free structured
// templates").
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace lamp {

constexpr int QUANT_THREADS = 512;

// One quantisation job: `outer` = batch*heads runs of L rows x D channels, blocks of `blk` rows.
// Variable-length batches (cu != null): run (b, h) is rows [cu[b], cu[b+1]) of head plane h of
// a [heads][total][D] tensor, at most L rows; scales stay [batch][heads][nb].
struct QuantJob {
  const uint16_t* x;
  uint8_t* codes;
  float* scales;
  int L, blk, nb;  // rows per run (varlen: the longest sequence), rows per block, blocks per run
  int blocks;      // outer * nb
  const int* cu;   // varlen: [batch + 1] row offsets, else null
  int heads, total;
};

__device__ __forceinline__ float h16_to_f32(uint32_t bits, bool bf16) {
  if (bf16) return __uint_as_float(bits << 16);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

// Lane-wise max(|a|, |b|) of two pairs of 16-bit floats (the sign bits of the result are
// meaningless; NaN lanes lose against numbers, as fmax does).
template <bool BF16>
__device__ __forceinline__ uint32_t absmax16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  if (BF16)
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  else
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Packed pairs of fp32 (lo in the low word).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// The two 16-bit values of a 32-bit word as a packed fp32 pair (exact).
template <bool BF16>
__device__ __forceinline__ uint64_t h2_to_f2(uint32_t w) {
  if (BF16) return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return f2pack(h16_to_f32(w & 0xFFFFu, false), h16_to_f32(w >> 16, false));
}

__device__ __forceinline__ float rcp_approx(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// The quotient x / s is estimated as x * rcp(s).  The estimate is within 1.5 * 2^-23 relative
// of the exact quotient z, and the IEEE quotient fl32(z) within 2^-24, so the estimate and
// fl32(z) round to the same code unless a rounding boundary of the 8-bit format lies within
// that distance of the estimate.  `near_*` flag estimates within a wider margin of a boundary
// (2^-12 absolute for INT8's half-integers, |q| <= 127.01; 64 units of the 20 dropped mantissa
// bits for E4M3's midpoints, and 2^-12 in units of 2^-9 on E4M3's uniform grid below 2^-6);
// those elements are recomputed with the IEEE divide.  (Below 2^-6, E4M3's uniform grid, the
// estimate is not tested: any non-zero element there takes the IEEE divide.)
__device__ __forceinline__ bool near_e4m3(float q) {
  const uint32_t b = __float_as_uint(q);
  // 20 dropped mantissa bits within 64 of the midpoint 0x80000 (normal e4m3 range) ...
  const bool mid = ((b - 0x7FFC0u) & 0xFFFFFu) <= 128u;
  // ... or 0 < |q| < 2^-6 (e4m3's subnormal range): always recomputed exactly.
  const bool sub = ((b & 0x7FFFFFFFu) - 1u) < 0x3C7FFFFFu;
  return mid || sub;
}

// Eight 16-bit inputs -> eight 8-bit codes (two 32-bit words), x / s as described above.
// INT8: t = fma(x, r, 1.5 * 2^23) rounds the exact product e = x * r once, to the integer
// rint(e) held in t's low mantissa bits (exact for |e| < 2^22), so t's low byte is the two's-
// complement code; d = fma(x, r, -(t - 1.5 * 2^23)) = e - rint(e), and the estimate is near a
// half-integer when |d| > 0.5 - 2^-12.  (e is within 2^-23 relative of x / s: one ulp of the
// reciprocal estimate, the product being exact inside the fma.)
template <bool BF16, bool E4M3>
__device__ __forceinline__ uint2 encode8(const uint4 w, float s, float r) {
  constexpr float MAGIC = 12582912.0f;  // 1.5 * 2^23
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  const uint64_t r2 = f2pack(r, r);
  uint32_t out[2];
  if (E4M3) {
    float q[8];
    bool nr = false;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f2unpack(f2mul(h2_to_f2<BF16>(ws[e]), r2), q[2 * e], q[2 * e + 1]);
      nr |= near_e4m3(q[2 * e]) | near_e4m3(q[2 * e + 1]);
    }
    if (nr) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        q[2 * e] = __fdiv_rn(h16_to_f32(ws[e] & 0xFFFFu, BF16), s);
        q[2 * e + 1] = __fdiv_rn(h16_to_f32(ws[e] >> 16, BF16), s);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
      out[h] = e4m3x2(q[4 * h], q[4 * h + 1]) | (e4m3x2(q[4 * h + 2], q[4 * h + 3]) << 16);
  } else {
    const uint64_t m2 = f2pack(MAGIC, MAGIC);
    float t[8];
    float dmax = 0.0f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint64_t x2 = h2_to_f2<BF16>(ws[e]);
      const uint64_t t2 = f2fma(x2, r2, m2);
      float d0, d1;
      f2unpack(f2fma(x2, r2, f2sub(m2, t2)), d0, d1);
      dmax = fmaxf(dmax, fmaxf(fabsf(d0), fabsf(d1)));
      f2unpack(t2, t[2 * e], t[2 * e + 1]);
    }
    if (dmax > 0.5f - 0x1.0p-12f) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        t[2 * e] = __fadd_rn(__fdiv_rn(h16_to_f32(ws[e] & 0xFFFFu, BF16), s), MAGIC);
        t[2 * e + 1] = __fadd_rn(__fdiv_rn(h16_to_f32(ws[e] >> 16, BF16), s), MAGIC);
      }
    }
    // |x| <= absmax and s = fl32(absmax / 127) give |fl32(x / s)| < 127.5: codes need no clamp.
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = __float_as_uint(t[e]);
#pragma unroll
    for (int h = 0; h < 2; ++h)
      out[h] = __byte_perm(__byte_perm(c[4 * h], c[4 * h + 1], 0x0040),
                           __byte_perm(c[4 * h + 2], c[4 * h + 3], 0x0040), 0x5410);
  }
  return make_uint2(out[0], out[1]);
}

// Eight 16-bit inputs -> codes with the IEEE divide for every element (blocks whose scale is
// subnormal: it carries few significant bits, so x / s can exceed 127.5 and INT8 is clamped).
template <bool BF16, bool E4M3>
__device__ __forceinline__ uint2 encode8_exact(const uint4 w, float s) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  uint32_t o2[2] = {0, 0};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x0 = __fdiv_rn(h16_to_f32(ws[e] & 0xFFFFu, BF16), s);
    const float x1 = __fdiv_rn(h16_to_f32(ws[e] >> 16, BF16), s);
    const int c0 = max(-127, min(127, __float2int_rn(x0)));
    const int c1 = max(-127, min(127, __float2int_rn(x1)));
    const uint32_t pair = E4M3 ? e4m3x2(x0, x1)
                               : ((static_cast<uint32_t>(c0) & 0xFFu) |
                                  ((static_cast<uint32_t>(c1) & 0xFFu) << 8));
    o2[e >> 1] |= pair << ((e & 1) * 16);
  }
  return make_uint2(o2[0], o2[1]);
}

// Pipeline shape for blocks of VEC 16-byte vectors per thread: NS shared-memory stages, each
// holding one whole block (the absmax needs the whole block before any code is written).
template <int VEC>
struct QuantPipe {
  static constexpr int STAGE_BYTES = VEC * QUANT_THREADS * 16;
  static constexpr int NS = STAGE_BYTES <= 8192 ? 4 : 3;
  // stages, then NS mbarriers, then NS block descriptors (QuantBlock, 32 bytes each)
  static constexpr int SMEM_BYTES = NS * STAGE_BYTES + NS * 8 + NS * 32;
  static constexpr int CTAS_PER_SM = STAGE_BYTES <= 8192 ? 4 : (STAGE_BYTES <= 32768 ? 2 : 1);
  static constexpr int MIN_CTAS = CTAS_PER_SM > 2 ? 2 : CTAS_PER_SM;  // register bound
};

// Where block `b` of the combined (Q, K) grid lives.
struct QuantBlock {
  const uint16_t* x;  // first input element of the block
  uint8_t* codes;     // first code of the block
  float* scale;       // the block's scale
  int nvec;           // 16-byte vectors in it (ragged last block of a run: fewer rows)
};
static_assert(sizeof(QuantBlock) == 32, "descriptor slot");
__device__ __forceinline__ QuantBlock quant_locate(const QuantJob& j0, const QuantJob& j1, int b,
                                                   int D) {
  const bool second = b >= j0.blocks;
  const int id = b - (second ? j0.blocks : 0);
  // (fields are selected one by one: a reference to a runtime-chosen kernel parameter would
  // copy both jobs to local memory)
  const int L = second ? j1.L : j0.L, blk = second ? j1.blk : j0.blk, nb = second ? j1.nb : j0.nb;
  const uint16_t* x = second ? j1.x : j0.x;
  uint8_t* codes = second ? j1.codes : j0.codes;
  float* scales = second ? j1.scales : j0.scales;
  const int* cu = second ? j1.cu : j0.cu;
  const int o = id / nb, bi = id - o * nb;
  const int r0 = bi * blk;
  if (cu) {  // rows of sequence o / heads in head plane o % heads, clipped to the tensor
    const int heads = second ? j1.heads : j0.heads, total = second ? j1.total : j0.total;
    const int sb = o / heads, h = o - sb * heads;
    const int s0 = min(max(__ldg(cu + sb), 0), total);
    const int len = min(max(__ldg(cu + sb + 1) - s0, 0), min(L, total - s0));
    const int rows = min(max(len - r0, 0), blk);
    const size_t base = (static_cast<size_t>(h) * total + s0 + min(r0, len)) * D;
    return QuantBlock{x + base, codes + base, scales + id, rows * D / 8};
  }
  const size_t base = (static_cast<size_t>(o) * L + r0) * D;
  return QuantBlock{x + base, codes + base, scales + id, min(blk, L - r0) * D / 8};
}

// Persistent CTAs; CTA c quantises blocks c, c + grid, c + 2 grid, ... of the combined grid
// (blocks [0, j0.blocks) are Q's, the rest K's).  Thread 0 keeps NS blocks in flight with bulk
// copies into the shared-memory ring; every thread moves its VEC vectors of the current block
// to registers, the CTA reduces the absmax (lane-wise 16-bit abs-max, then an integer max of the
// magnitude bits, which orders non-NaN fp16/bf16 values by |x|), the stage is refilled at once, and the codes are computed
// from registers and written with 8-byte stores.  Every wait is bounded: a timeout sets the
// device error word, the CTA waits (bounded) for its copies still in flight and returns.
template <bool BF16, bool E4M3, int VEC>
__global__ void __launch_bounds__(QUANT_THREADS, QuantPipe<VEC>::MIN_CTAS)
    quant_kernel(const QuantJob j0, const QuantJob j1, int D, uint32_t wait_us) {
  using P = QuantPipe<VEC>;
  extern __shared__ __align__(128) uint8_t qsm[];
  uint64_t* full = reinterpret_cast<uint64_t*>(qsm + P::NS * P::STAGE_BYTES);
  // Block descriptors, written by the issuing thread before the copy's arrival on full[]:
  // the other threads read them after their wait, so the index arithmetic runs once per block.
  QuantBlock* desc = reinterpret_cast<QuantBlock*>(qsm + P::NS * P::STAGE_BYTES + P::NS * 8);
  __shared__ uint32_t red[2][QUANT_THREADS / 32];
  __shared__ uint32_t abort_word;
  const int total = j0.blocks + j1.blocks;
  const int stride = static_cast<int>(gridDim.x);
  const int first = static_cast<int>(blockIdx.x);
  const int mine = first < total ? (total - first + stride - 1) / stride : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P::NS; ++s) mbar_init(&full[s], 1);
    abort_word = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  auto issue = [&](int i) {  // the CTA's i-th block into stage i % NS
    const QuantBlock qb = quant_locate(j0, j1, first + i * stride, D);
    desc[i % P::NS] = qb;
    const uint32_t bytes = static_cast<uint32_t>(qb.nvec) * 16u;
    uint64_t* bar = &full[i % P::NS];
    mbar_arrive_expect_tx(bar, bytes);
    // (an empty block -- past the end of a short sequence -- completes on the arrival alone)
    if (bytes) bulk_load(smem_u32(qsm + (i % P::NS) * P::STAGE_BYTES), qb.x, bytes, bar);
  };
  if (threadIdx.x == 0)
    for (int i = 0; i < P::NS && i < mine; ++i) issue(i);

  const WaitCtx wc{smem_u32(&abort_word), wait_us};
  int i = 0;
  for (; i < mine; ++i) {
    const int st = i % P::NS;
    const bool ok = mbar_wait(&full[st], (i / P::NS) & 1u, wc, 0x40u);
    const QuantBlock qb = desc[st];
    const uint4* src = reinterpret_cast<const uint4*>(qsm + st * P::STAGE_BYTES);
    uint4 buf[VEC];
    uint32_t m2 = 0;
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const int v = threadIdx.x + k * QUANT_THREADS;
      buf[k] = v < qb.nvec ? src[v] : make_uint4(0, 0, 0, 0);
      m2 = absmax16x2<BF16>(m2, absmax16x2<BF16>(buf[k].x, buf[k].y));
      m2 = absmax16x2<BF16>(m2, absmax16x2<BF16>(buf[k].z, buf[k].w));
    }
    // |x| orders like the magnitude bits as unsigned integers (non-NaN fp16 / bf16)
    m2 &= 0x7FFF7FFFu;
    uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    if ((threadIdx.x & 31) == 0) red[i & 1][threadIdx.x >> 5] = mb;
    // Every thread has its data in registers and its partial max in red[]: the stage is free.
    if (!__syncthreads_and(ok)) break;
    if (threadIdx.x == 0 && i + P::NS < mine) issue(i + P::NS);
    // every warp reduces the 16 warp maxima itself (no second barrier)
    mb = __reduce_max_sync(0xFFFFFFFFu, red[i & 1][threadIdx.x & (QUANT_THREADS / 32 - 1)]);
    const float amax = h16_to_f32(mb, BF16);
    const float s = (amax == 0.0f) ? 0.0f : __fdiv_rn(amax, E4M3 ? 448.0f : 127.0f);
    if (threadIdx.x == 0) *qb.scale = s;
    // The reciprocal estimate needs a normal s: a block whose scale is subnormal (absmax below
    // about 1.5e-36) takes the IEEE divide for every element.
    const bool tiny = s < 0x1.0p-126f;
    const float r = tiny ? 0.0f : rcp_approx(s);
    uint2* cv = reinterpret_cast<uint2*>(qb.codes);
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const int v = threadIdx.x + k * QUANT_THREADS;
      if (v < qb.nvec) {
        uint2 out = make_uint2(0, 0);
        if (s != 0.0f)
          out = tiny ? encode8_exact<BF16, E4M3>(buf[k], s) : encode8<BF16, E4M3>(buf[k], s, r);
        cv[v] = out;
      }
    }
  }
  if (i < mine && threadIdx.x == 0) {
    // Gave up on block i: wait (bounded, no abort word) for the copies still in flight.
    const int issued = min(mine, i + P::NS);
    for (int d = i; d < issued; ++d)
      if (!mbar_wait(&full[d % P::NS], (d / P::NS) & 1u, WaitCtx{0u, wait_us}, 0x41u)) break;
  }
}

// SplitMix64 step from state x: add the golden gamma, then the variant-13 finaliser.
__device__ __forceinline__ uint64_t splitmix64_step(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ------------------------------------------------------------------ 8-bit V -----------
// Per-channel E4M3 V for the 8-bit P.V mode (LampAttention abstract, exponentials in 8-bit
// formats; the pages give no V format): one scale per (batch, KV head, channel) over all keys,
// s = fl32(a / 448) with a the channel's absolute maximum, code = E4M3(fl32(v / s)) rounded to
// nearest even; a = 0 gives s = 0 and zero codes.  Codes channel-major [planes][D][Lk_pad]
// (keys contiguous, Lk_pad = Lk rounded up to 16, the padding zero), so that a tile of 128
// keys is a K-major operand of the P.V MMA.
//
// Pass 1: the channel maxima, folded into amax[planes][D] as bit patterns (non-negative floats
// order as their bits; the array starts at zero).  Block = D threads (thread = channel),
// grid = (key chunks of VQ_KEYS, planes).
constexpr int VQ_KEYS = 256;

template <bool BF16>
__global__ void vmax_kernel(const uint16_t* __restrict__ v, uint32_t* __restrict__ amax, int Lk,
                            int D) {
  const int d = threadIdx.x, plane = blockIdx.y;
  const int j0 = blockIdx.x * VQ_KEYS, j1 = min(Lk, j0 + VQ_KEYS);
  const uint16_t* src = v + static_cast<size_t>(plane) * Lk * D + d;
  float a = 0.0f;
  for (int j = j0; j < j1; ++j) a = fmaxf(a, fabsf(h16_to_f32(src[static_cast<size_t>(j) * D], BF16)));
  atomicMax(amax + static_cast<size_t>(plane) * D + d, __float_as_uint(a));
}

// Pass 2: codes of 128 keys x D channels per CTA (256 threads), transposed through shared
// memory (words of 4 keys, rows padded to 33 words) and written as 128-byte channel rows.
template <bool BF16>
__global__ void vquant_kernel(const uint16_t* __restrict__ v, const uint32_t* __restrict__ amax,
                              uint8_t* __restrict__ v8t, int Lk, int Lk_pad, int D) {
  __shared__ uint32_t tw[256 * 33];  // [D][32 words] (+1 pad), D <= 256
  const int plane = blockIdx.y, j0 = blockIdx.x * 128;
  const uint16_t* src = v + static_cast<size_t>(plane) * Lk * D;
  for (int idx = threadIdx.x; idx < D * 32; idx += blockDim.x) {
    const int d = idx % D, wq = idx / D;  // channel, word of 4 keys
    const float a = __uint_as_float(__ldg(amax + static_cast<size_t>(plane) * D + d));
    const float sc = __fdiv_rn(a, 448.0f);
    uint32_t word = 0;
    if (a > 0.0f) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + 4 * wq + e;
        x[e] = (j < Lk) ? __fdiv_rn(h16_to_f32(src[static_cast<size_t>(j) * D + d], BF16), sc) : 0.0f;
      }
      word = e4m3x2(x[0], x[1]) | (e4m3x2(x[2], x[3]) << 16);
    }
    tw[d * 33 + wq] = word;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int d = warp; d < D; d += blockDim.x >> 5) {
    const int j = j0 + 4 * lane;
    if (j < Lk_pad)
      *reinterpret_cast<uint32_t*>(v8t + (static_cast<size_t>(plane) * D + d) * Lk_pad + j) =
          tw[d * 33 + lane];
  }
}

// Pass 3: the maxima become the scales (in place).
__global__ void vscale_kernel(uint32_t* __restrict__ amax_to_scale, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = __uint_as_float(amax_to_scale[i]);
    amax_to_scale[i] = __float_as_uint(a > 0.0f ? __fdiv_rn(a, 448.0f) : 0.0f);
  }
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

// Structured static template: one thread per mask word.  Row qt's diagonal key tile is the
// tile of the key aligned with its last query row (bottom-right); group g is 16-bit (bit 0)
// iff g < sink, |gd - g| < band, or stride > 0 divides |gd - g|.
__global__ void mask_template_kernel(uint64_t* __restrict__ mask, long long rows, int nqt,
                                     int ng, int W, int Lq, int Lk, int bm, int bn, int nkt,
                                     int group_tiles, int sink, int band, int stride) {
  const long long total = rows * W;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / W;
    const int w = static_cast<int>(i - row * W);
    const int qt = static_cast<int>(row % nqt);
    const long long aligned = static_cast<long long>(min(Lq, (qt + 1) * bm)) - 1 + Lk - Lq;
    const long long kd = aligned < 0 ? 0 : min(aligned / bn, static_cast<long long>(nkt - 1));
    const long long gd = kd / group_tiles;
    uint64_t word = 0;
    for (int bit = 0; bit < 64; ++bit) {
      const int g = w * 64 + bit;
      if (g >= ng) break;
      const long long d = gd >= g ? gd - g : g - gd;
      const bool sixteen = g < sink || d < band || (stride > 0 && d % stride == 0);
      if (!sixteen) word |= 1ull << bit;
    }
    mask[i] = word;
  }
}

}  // namespace lamp
