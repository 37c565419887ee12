// Tensor-core throughput probe (measurement only: the attention kernel's roofline is stated
// against tensor-core rates, and this kernel measures the rate of the MMA shapes that kernel
// issues).  One CTA per SM; its elected thread issues `iters` x 8 back-to-back tcgen05 MMAs
// (M = 128, N = the template's N) into one TMEM accumulator, then waits for completion.  The
// shared-memory descriptors are built once and advanced by constant offsets, so the issuing
// thread spends a few instructions per MMA and the tensor core, not the issue loop, sets the
// pace.  Operands are zero: only the time is of interest.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace lamp {

enum ProbeKind : int {
  PROBE_F16_SS = 0,  // kind::f16 (bf16), A and B from shared memory, K = 16 per MMA
  PROBE_I8_SS = 1,   // kind::i8, A and B from shared memory, K = 32 per MMA
  PROBE_F16_TS = 2,  // kind::f16 (bf16), A from tensor memory, B from shared memory
};

constexpr int PROBE_THREADS = 128;
constexpr int PROBE_A_BYTES = 128 * 128;  // 128 rows x 128 bytes, 128-byte swizzle
constexpr int PROBE_B_BYTES = 256 * 128;  // up to N = 256 rows
constexpr int PROBE_SMEM = PROBE_A_BYTES + PROBE_B_BYTES + 1024 + 64;

template <int KIND, int N>
__global__ void __launch_bounds__(PROBE_THREADS, 1)
    mma_probe_kernel(int iters, uint32_t wait_us) {
  extern __shared__ uint8_t probe_raw[];
  const uint32_t raw = smem_u32(probe_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned operand base
  uint8_t* sbase = probe_raw + (base - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sbase + PROBE_A_BYTES + PROBE_B_BYTES);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  uint32_t* abort_word = tslot + 1;
  const int warp = threadIdx.x >> 5;

  for (int i = threadIdx.x; i < (PROBE_A_BYTES + PROBE_B_BYTES) / 16; i += PROBE_THREADS)
    reinterpret_cast<uint4*>(sbase)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_word = 0;
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();  // zeros written by threads, read by the tensor core
  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (KIND == PROBE_F16_TS) {  // zero A: 128 lanes x 64 columns at column 256
    uint32_t z[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) z[e] = 0u;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_st16(lane_base + 256 + c * 16, z);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (threadIdx.x == 0) {
    constexpr uint32_t id = (KIND == PROBE_I8_SS) ? idesc(2, 1, 1, 0, 0, N, 128)
                                                  : idesc(1, 1, 1, 0, 0, N, 128);
    const uint64_t a0 = sdesc(base, 16, 1024, SWZ_128B);
    const uint64_t b0 = sdesc(base + PROBE_A_BYTES, 16, 1024, SWZ_128B);
    // each MMA step moves 32 bytes along K inside the 128-byte swizzled row: +2 in the
    // descriptor's 16-byte address field; two groups of four steps cover two K blocks
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint64_t koff = static_cast<uint64_t>((s & 3) * 2);
        const uint32_t acc = (it > 0 || s > 0) ? 1u : 0u;
        if (KIND == PROBE_I8_SS)
          mma_i8_ss(tbase, a0 + koff, b0 + koff, id, acc);
        else if (KIND == PROBE_F16_SS)
          mma_f16_ss(tbase, a0 + koff, b0 + koff, id, acc);
        else
          mma_f16_ts(tbase, tbase + 256 + s * 8, b0 + koff, id, acc);
      }
    }
    tc_commit(bar);
    mbar_wait(bar, 0, WaitCtx{smem_u32(abort_word), wait_us}, 0x50u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace lamp
