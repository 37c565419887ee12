// Host side of the C ABI declared in include/lamp.h: argument checks, TMA tensor maps,
// workspace management and kernel launches.  All device code is included into this one
// translation unit so that the device error word is a single file-scope symbol.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/lamp.h"
#include "attn_fwd.cuh"
#include "attn_fwd_pp.cuh"
#include "decode.cuh"
#include "mma_probe.cuh"
#include "quant.cuh"

// Scratch of lamp_attn_fwd_noalloc: a file-scope device array that every GPU loading this
// library holds until the process exits.  In host code the symbol is only a stand-in; its
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[LAMP_NOALLOC_MAX_BYTES];

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(LAMP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define LAMP_CUDA(call, what)                  \
  do {                                         \
    cudaError_t e_ = (call);                   \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// O is written with 32-byte stores
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

int tile_shape(int D, int* bm, int* bn) {
  if (D == 64) { *bm = 64; *bn = 64; return LAMP_OK; }
  if (D == 128) { *bm = 128; *bn = 128; return LAMP_OK; }
  if (D == 256) { *bm = 64; *bn = 128; return LAMP_OK; }
  return LAMP_ERR_UNSUPPORTED;
}

int check_sizes(int B, int H, int Hkv, int Lq, int Lk, int D) {
  if (B < 1 || H < 1 || Hkv < 1 || Lq < 1 || Lk < 1)
    return fail(LAMP_ERR_INVALID, "sizes must be positive (B=%d H=%d Hkv=%d Lq=%d Lk=%d)", B, H,
                Hkv, Lq, Lk);
  if (H % Hkv != 0) return fail(LAMP_ERR_INVALID, "H (%d) must be a multiple of Hkv (%d)", H, Hkv);
  int bm, bn;
  if (tile_shape(D, &bm, &bn) != LAMP_OK)
    return fail(LAMP_ERR_UNSUPPORTED, "head dimension D=%d not supported (64, 128, 256)", D);
  if (static_cast<long long>(B) * H * Lq * D >= (1ll << 40) ||
      static_cast<long long>(B) * H > (1 << 24) || Lq > (1 << 30) || Lk > (1 << 30))
    return fail(LAMP_ERR_INVALID, "problem too large");
  return LAMP_OK;
}

// ---------------------------------------------------------------- tensor maps ---------

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_mu;

int get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return LAMP_OK;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(LAMP_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return LAMP_OK;
}

// 3-D map over [outer][L][D] elements of `ebytes` bytes; box (inner, rows, 1).
int make_map(CUtensorMap* m, const void* base, int ebytes, int D, int L, int outer, int inner,
             int rows, CUtensorMapSwizzle swz) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * ebytes,
                           static_cast<cuuint64_t>(D) * L * ebytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, ebytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LAMP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LAMP_OK;
}

// 3-D map over 8-bit [outer][rows][inner] with a row pitch of `pitch` bytes (>= inner, a
// multiple of 16); box (box_inner, box_rows, 1).
int make_map_pitch(CUtensorMap* m, const void* base, int inner, int pitch, int rows, int outer,
                   int box_inner, int box_rows, CUtensorMapSwizzle swz) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(pitch),
                           static_cast<cuuint64_t>(pitch) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LAMP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return LAMP_OK;
}

// Row pitch of the channel-major 8-bit V: keys rounded up to 16 bytes.
int v8_pitch(int Lk) { return (Lk + 15) & ~15; }

// ---------------------------------------------------------------- workspace -----------

struct Workspace {
  void* user = nullptr;
  size_t user_bytes = 0;
  void* cached[64] = {};
  size_t cached_bytes[64] = {};
};
Workspace g_ws;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
  size_t q8, k8, qs, ks, v8, vs, total;  // v8, vs: the 8-bit P.V mode's V codes and scales
};

// q_rows / k_rows: rows per head plane of a variable-length batch (0: dense, B * L).
WsLayout ws_layout(int B, int H, int Hkv, int Lq, int Lk, int D, int q_rows = 0, int k_rows = 0,
                   bool pv8 = false) {
  int bm, bn;
  tile_shape(D, &bm, &bn);
  const size_t nqt = (Lq + bm - 1) / bm, nkt = (Lk + bn - 1) / bn;
  const size_t qr = q_rows ? static_cast<size_t>(q_rows) : static_cast<size_t>(B) * Lq;
  const size_t kr = k_rows ? static_cast<size_t>(k_rows) : static_cast<size_t>(B) * Lk;
  WsLayout w;
  w.q8 = 0;
  w.k8 = align256(qr * H * D);
  w.qs = w.k8 + align256(kr * Hkv * D);
  w.ks = w.qs + align256(static_cast<size_t>(B) * H * nqt * sizeof(float));
  w.v8 = w.ks + align256(static_cast<size_t>(B) * Hkv * nkt * sizeof(float));
  w.vs = w.v8 + (pv8 ? align256(static_cast<size_t>(B) * Hkv * D * v8_pitch(Lk)) : 0);
  w.total = w.vs + (pv8 ? align256(static_cast<size_t>(B) * Hkv * D * sizeof(float)) : 0);
  return w;
}

// The cached workspace of the current device, grown in stream order on `st` (the old block is
// released with cudaFreeAsync behind the work already queued on `st`, the new one allocated
// with cudaMallocAsync), so that growing it never synchronises the device.
int get_workspace(size_t need, cudaStream_t st, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ws.user) {
    if (g_ws.user_bytes < need)
      return fail(LAMP_ERR_INVALID, "workspace too small: %zu bytes set, %zu needed", g_ws.user_bytes, need);
    *out = g_ws.user;
    return LAMP_OK;
  }
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_INVALID, "device index out of range");
  if (g_ws.cached_bytes[dev] < need) {
    void* p = nullptr;
    LAMP_CUDA(cudaMallocAsync(&p, need, st), "cudaMallocAsync(workspace)");
    if (g_ws.cached[dev]) cudaFreeAsync(g_ws.cached[dev], st);
    g_ws.cached[dev] = p;
    g_ws.cached_bytes[dev] = need;
  }
  *out = g_ws.cached[dev];
  return LAMP_OK;
}

// ---------------------------------------------------------------- launches ------------

constexpr uint32_t kWaitUs = 2000000u;  // 2 s per wait: far beyond any legitimate stall

int sm_count(int* n) {
  static int cached[64] = {};
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_CUDA, "device index out of range");
  if (!cached[dev])
    LAMP_CUDA(cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev),
              "cudaDeviceGetAttribute(multiProcessorCount)");
  *n = cached[dev];
  return LAMP_OK;
}

template <bool BF16, bool E4M3, int VEC>
int launch_quant_v(const lamp::QuantJob& j0, const lamp::QuantJob& j1, int D, cudaStream_t st) {
  using P = lamp::QuantPipe<VEC>;
  static bool attr_set[64] = {};
  int dev = 0, nsm = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (int r = sm_count(&nsm)) return r;
  if (!attr_set[dev]) {
    LAMP_CUDA(cudaFuncSetAttribute(lamp::quant_kernel<BF16, E4M3, VEC>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM_BYTES),
              "cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  const int total = j0.blocks + j1.blocks;
  const int grid = std::min(total, nsm * P::CTAS_PER_SM);
  lamp::quant_kernel<BF16, E4M3, VEC>
      <<<grid, lamp::QUANT_THREADS, P::SMEM_BYTES, st>>>(j0, j1, D, kWaitUs);
  LAMP_CUDA(cudaGetLastError(), "quant_kernel launch");
  return LAMP_OK;
}

template <bool BF16, bool E4M3>
int launch_quant_t(const lamp::QuantJob& j0, const lamp::QuantJob& j1, int D, int vec,
                   cudaStream_t st) {
  if (vec <= 1) return launch_quant_v<BF16, E4M3, 1>(j0, j1, D, st);
  if (vec <= 4) return launch_quant_v<BF16, E4M3, 4>(j0, j1, D, st);
  return launch_quant_v<BF16, E4M3, 8>(j0, j1, D, st);
}

// Job for `outer` runs of L rows in blocks of blk rows; an empty job when x is NULL.
int quant_job(const void* x, void* codes, float* scales, int outer, int L, int blk,
              lamp::QuantJob* j) {
  *j = lamp::QuantJob{static_cast<const uint16_t*>(x), static_cast<uint8_t*>(codes), scales, L,
                      blk, (L + blk - 1) / blk, 0, nullptr, 0, 0};
  if (!x) return LAMP_OK;
  const long long blocks = static_cast<long long>(outer) * j->nb;
  if (blocks > 0x3FFFFFFF) return fail(LAMP_ERR_INVALID, "too many quantisation blocks");
  j->blocks = static_cast<int>(blocks);
  return LAMP_OK;
}

// Variable-length batch: run (b, h) is sequence b of head plane h, cu the row offsets.
void varlen_job(lamp::QuantJob* j, const int* cu, int heads, int total) {
  if (!j->x) return;
  j->cu = cu;
  j->heads = heads;
  j->total = total;
}

int quant_qk(const void* q, const void* k, void* q8, void* k8, float* q_scale, float* k_scale,
             int B, int H, int Hkv, int Lq, int Lk, int D, int mode, cudaStream_t st,
             const int* cu_q = nullptr, const int* cu_k = nullptr, int total_q = 0,
             int total_k = 0) {
  int bm, bn;
  tile_shape(D, &bm, &bn);
  const bool bf16 = (mode & LAMP_IN_BF16) != 0, e4m3 = (mode & LAMP_FMT_E4M3) != 0;
  lamp::QuantJob jq, jk;
  if (int r = quant_job(q, q8, q_scale, B * H, Lq, bm, &jq)) return r;
  if (int r = quant_job(k, k8, k_scale, B * Hkv, Lk, bn, &jk)) return r;
  if (cu_q) varlen_job(&jq, cu_q, H, total_q);
  if (cu_k) varlen_job(&jk, cu_k, Hkv, total_k);
  if (jq.blocks + jk.blocks == 0) return LAMP_OK;
  // 16-byte vectors per thread for the larger block
  const int vec = (std::max(q ? bm : 0, k ? bn : 0) * D / 8 + lamp::QUANT_THREADS - 1) /
                  lamp::QUANT_THREADS;
  if (bf16 && e4m3) return launch_quant_t<true, true>(jq, jk, D, vec, st);
  if (bf16) return launch_quant_t<true, false>(jq, jk, D, vec, st);
  if (e4m3) return launch_quant_t<false, true>(jq, jk, D, vec, st);
  return launch_quant_t<false, false>(jq, jk, D, vec, st);
}

// Per-channel 8-bit V (the 8-bit P.V mode): maxima into v_scale (as bits), codes, scales.
int quant_v(const void* v, void* v8t, float* v_scale, int B, int Hkv, int Lk, int D, int mode,
            cudaStream_t st) {
  const int planes = B * Hkv;
  const bool bf16 = (mode & LAMP_IN_BF16) != 0;
  auto* amax = reinterpret_cast<uint32_t*>(v_scale);
  const auto* src = static_cast<const uint16_t*>(v);
  auto* dst = static_cast<uint8_t*>(v8t);
  LAMP_CUDA(cudaMemsetAsync(amax, 0, static_cast<size_t>(planes) * D * sizeof(float), st),
            "memset V maxima");
  const dim3 g1((Lk + lamp::VQ_KEYS - 1) / lamp::VQ_KEYS, planes);
  if (bf16) lamp::vmax_kernel<true><<<g1, D, 0, st>>>(src, amax, Lk, D);
  else lamp::vmax_kernel<false><<<g1, D, 0, st>>>(src, amax, Lk, D);
  LAMP_CUDA(cudaGetLastError(), "vmax_kernel launch");
  const int pitch = v8_pitch(Lk);
  const dim3 g2((pitch + 127) / 128, planes);
  if (bf16) lamp::vquant_kernel<true><<<g2, 256, 0, st>>>(src, amax, dst, Lk, pitch, D);
  else lamp::vquant_kernel<false><<<g2, 256, 0, st>>>(src, amax, dst, Lk, pitch, D);
  LAMP_CUDA(cudaGetLastError(), "vquant_kernel launch");
  const int n = planes * D;
  lamp::vscale_kernel<<<(n + 255) / 256, 256, 0, st>>>(amax, n);
  LAMP_CUDA(cudaGetLastError(), "vscale_kernel launch");
  return LAMP_OK;
}

template <class C, bool BF16, bool E4M3, bool SKIP, bool DBG = false>
int launch_attn_cfg_t(const lamp::AttnParams& p, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    LAMP_CUDA(cudaFuncSetAttribute(lamp::attn_fwd_kernel<C, BF16, E4M3, SKIP, DBG>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES),
              "cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  lamp::attn_fwd_kernel<C, BF16, E4M3, SKIP, DBG><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(p);
  LAMP_CUDA(cudaGetLastError(), "attn_fwd_kernel launch");
  return LAMP_OK;
}

template <class C>
int launch_attn_cfg(const lamp::AttnParams& p, int grid, cudaStream_t st) {
  // the debug capture has its own instantiations (lamp_attn_debug: no threshold skip)
  if (p.dbg_slot) {
    if (p.bf16) return p.e4m3 ? launch_attn_cfg_t<C, true, true, false, true>(p, grid, st)
                              : launch_attn_cfg_t<C, true, false, false, true>(p, grid, st);
    return p.e4m3 ? launch_attn_cfg_t<C, false, true, false, true>(p, grid, st)
                  : launch_attn_cfg_t<C, false, false, false, true>(p, grid, st);
  }
  // the threshold skip has its own instantiation, so that the look-ahead path without it keeps
  // its code
  if (!std::isinf(p.skip_log2)) {
    if (p.bf16) return p.e4m3 ? launch_attn_cfg_t<C, true, true, true>(p, grid, st)
                              : launch_attn_cfg_t<C, true, false, true>(p, grid, st);
    return p.e4m3 ? launch_attn_cfg_t<C, false, true, true>(p, grid, st)
                  : launch_attn_cfg_t<C, false, false, true>(p, grid, st);
  }
  if (p.bf16) return p.e4m3 ? launch_attn_cfg_t<C, true, true, false>(p, grid, st)
                            : launch_attn_cfg_t<C, true, false, false>(p, grid, st);
  return p.e4m3 ? launch_attn_cfg_t<C, false, true, false>(p, grid, st)
                : launch_attn_cfg_t<C, false, false, false>(p, grid, st);
}

template <bool BF16, bool ADAPTIVE, bool VARLEN, bool DBG = false, bool TK = false>
int launch_attn_pp_t(const lamp::AttnParams& p, int grid, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    LAMP_CUDA(cudaFuncSetAttribute(lamp::attn_fwd_pp_kernel<BF16, ADAPTIVE, VARLEN, DBG, TK>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   lamp::PPCfg::SMEM_BYTES),
              "cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  lamp::attn_fwd_pp_kernel<BF16, ADAPTIVE, VARLEN, DBG, TK>
      <<<grid, lamp::PPCfg::THREADS, lamp::PPCfg::SMEM_BYTES, st>>>(p);
  LAMP_CUDA(cudaGetLastError(), "attn_fwd_pp_kernel launch");
  return LAMP_OK;
}

template <bool VARLEN>
int launch_attn_pp_v(const lamp::AttnParams& p, int grid, cudaStream_t st) {
  if (p.bf16) return p.adaptive ? launch_attn_pp_t<true, true, VARLEN>(p, grid, st)
                                : launch_attn_pp_t<true, false, VARLEN>(p, grid, st);
  return p.adaptive ? launch_attn_pp_t<false, true, VARLEN>(p, grid, st)
                    : launch_attn_pp_t<false, false, VARLEN>(p, grid, st);
}

// Scheduler slots of the two-tile kernel, handed out round-robin per device.  A launch's tag
// is the number of earlier launches given the same slot, plus one: distinct among the launches
// that share a slot (and never 0, the idle value).
std::mutex g_sched_mu;
unsigned long long* g_sched_base[64] = {};
uint32_t g_sched_seq[64] = {};

int sched_base(unsigned long long** out) {
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_INVALID, "device index out of range");
  if (!g_sched_base[dev]) {
    void* a = nullptr;
    LAMP_CUDA(cudaGetSymbolAddress(&a, lamp::g_lamp_sched), "cudaGetSymbolAddress(sched)");
    if (!a) return fail(LAMP_ERR_CUDA, "scheduler slots have no device address");
    g_sched_base[dev] = static_cast<unsigned long long*>(a);
  }
  *out = g_sched_base[dev];
  return LAMP_OK;
}

int sched_slot(unsigned long long** slot, uint32_t* tag) {
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_sched_mu);
  unsigned long long* base = nullptr;
  if (int r = sched_base(&base)) return r;
  const uint32_t s = g_sched_seq[dev]++;
  *slot = base + (s % lamp::SCHED_SLOTS);
  *tag = s / lamp::SCHED_SLOTS + 1u;
  return LAMP_OK;
}

// Variable-length batches have their own instantiation: the dense one keeps compile-time
// zero offsets.  The debug capture (dense batches only) has its own as well, and so has the
// ticket counter (dense batches only).  The debug capture always takes the fixed order (its
// outputs do not depend on the order).
int launch_attn_pp(const lamp::AttnParams& p0, int grid, bool dynamic, cudaStream_t st) {
  lamp::AttnParams p = p0;
  p.sched = nullptr;
  p.sched_tag = 0;
  if (p.dbg_slot) {
    if (p.bf16) return p.adaptive ? launch_attn_pp_t<true, true, false, true>(p, grid, st)
                                  : launch_attn_pp_t<true, false, false, true>(p, grid, st);
    return p.adaptive ? launch_attn_pp_t<false, true, false, true>(p, grid, st)
                      : launch_attn_pp_t<false, false, false, true>(p, grid, st);
  }
  if (p.cu_q) return launch_attn_pp_v<true>(p, grid, st);
  if (!dynamic) return launch_attn_pp_v<false>(p, grid, st);
  if (int r = sched_slot(&p.sched, &p.sched_tag)) return r;
  if (p.bf16) return p.adaptive ? launch_attn_pp_t<true, true, false, false, true>(p, grid, st)
                                : launch_attn_pp_t<true, false, false, false, true>(p, grid, st);
  return p.adaptive ? launch_attn_pp_t<false, true, false, false, true>(p, grid, st)
                    : launch_attn_pp_t<false, false, false, false, true>(p, grid, st);
}

using Cfg64 = lamp::AttnCfg<64, 64, true>;
using Cfg128 = lamp::AttnCfg<128, 128, false>;
using Cfg256 = lamp::AttnCfg<256, 128, true>;
using Cfg128P8 = lamp::AttnCfg<128, 128, false, true>;  // 8-bit exponentials and P.V

int launch_attn_pv8(const lamp::AttnParams& p, int grid, cudaStream_t st) {
  if (p.bf16) return p.e4m3 ? launch_attn_cfg_t<Cfg128P8, true, true, false>(p, grid, st)
                            : launch_attn_cfg_t<Cfg128P8, true, false, false>(p, grid, st);
  return p.e4m3 ? launch_attn_cfg_t<Cfg128P8, false, true, false>(p, grid, st)
                : launch_attn_cfg_t<Cfg128P8, false, false, false>(p, grid, st);
}

// Host-side checks of a routed-attention call (sizes, operand pointers and alignment, causal /
// window, mode bits, group size, tau, scale, threshold skip).  Makes no CUDA call and enqueues
// nothing, so that every entry point can run all of them before it touches the workspace or
// launches a kernel.  q8 / k8 / q_scale / k_scale are checked only when `codes` is set (the
// end-to-end entry points place them in the workspace).  cu_q / cu_k non-null: variable-length
// batch of B sequences (at most Lq / Lk rows each) packed into [heads][total][D] tensors.
int check_attn(const void* q, const void* k, const void* v, bool codes, const void* q8,
               const void* k8, const float* q_scale, const float* k_scale, const void* o, int B,
               int H, int Hkv, int Lq, int Lk, int D, int causal, int window, float scale,
               int group_tiles, int mode, float tau, const int* cu_q, const int* cu_k,
               int total_q, int total_k, float skip_tau) {
  int r = check_sizes(B, H, Hkv, Lq, Lk, D);
  if (r) return r;
  const bool varlen = cu_q != nullptr;
  if (varlen && (!cu_k || total_q < 1 || total_k < 1 || total_q > (1 << 30) || total_k > (1 << 30)))
    return fail(LAMP_ERR_INVALID, "variable-length batch needs cu_q, cu_k and positive totals");
  if (!q || !k || !v || !o) return fail(LAMP_ERR_INVALID, "null operand pointer");
  if (codes && (!q8 || !k8 || !q_scale || !k_scale))
    return fail(LAMP_ERR_INVALID, "null 8-bit operand or scale pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned32(o) ||
      (codes && (!aligned16(q8) || !aligned16(k8))))
    return fail(LAMP_ERR_INVALID, "q, k, v, q8, k8 must be 16-byte and o 32-byte aligned");
  if (causal != 0 && causal != 1) return fail(LAMP_ERR_INVALID, "causal must be 0 or 1");
  if (window < 0) return fail(LAMP_ERR_INVALID, "window must be >= 0");
  if (window > 0 && !causal)
    return fail(LAMP_ERR_UNSUPPORTED, "a sliding window needs causal = 1");
  if ((mode & ~0x1Fu) != 0) return fail(LAMP_ERR_INVALID, "unknown mode bits 0x%x", mode);
  const bool adaptive = (mode & LAMP_ROUTE_ADAPTIVE) != 0;
  if (!adaptive && group_tiles < 1) return fail(LAMP_ERR_INVALID, "group_tiles must be >= 1");
  if (adaptive && !(tau == tau)) return fail(LAMP_ERR_INVALID, "tau is NaN");
  if (!(scale == scale)) return fail(LAMP_ERR_INVALID, "scale is NaN");
  const bool skip = !std::isinf(skip_tau) || skip_tau < 0.0f;
  if (skip && (!adaptive || !(skip_tau >= tau) || !(skip_tau >= 0.0f)))
    return fail(LAMP_ERR_INVALID, "skip_tau needs look-ahead mode and tau <= skip_tau");
  if ((mode & LAMP_PV_E4M3) && (D != 128 || varlen || skip))
    return fail(LAMP_ERR_UNSUPPORTED,
                "8-bit P.V: D = 128, dense batches and no threshold skip only");
  const long long grid = static_cast<long long>(B) * H * ((Lq + 127) / 128);
  if (grid > 0x7FFFFFFF) return fail(LAMP_ERR_INVALID, "grid too large");
  return LAMP_OK;
}

// Which attention kernel runs a prepared call.
enum AttnKernel { K_CFG64, K_PP, K_CFG128, K_CFG256, K_CFG128P8 };

struct AttnCall {
  lamp::AttnParams p;
  AttnKernel kernel;
  bool pp_dynamic;  // two-tile kernel: work items from a ticket counter (else a fixed order)
  int grid;
  size_t route_bytes;  // bytes of route_out cleared before the launch (0: none)
};

// Tensor maps and kernel parameters of a call that passed check_attn (host work only: nothing
// is enqueued; a failure here leaves the device untouched).
int prepare_attn(const void* q, const void* k, const void* v, const void* q8, const void* k8,
                 const float* q_scale, const float* k_scale, void* o, float* lse, int B, int H,
                 int Hkv, int Lq, int Lk, int D, int causal, int window, float scale,
                 const uint64_t* mask_bits, int group_tiles, int mode, float tau,
                 uint8_t* route_out, const int* cu_q, const int* cu_k, int total_q, int total_k,
                 float skip_tau, AttnCall* call, const float* v_scale = nullptr) {
  int r;
  if ((r = get_encode())) return r;
  const bool pv8 = (mode & LAMP_PV_E4M3) != 0;  // v is then the channel-major 8-bit V
  const bool varlen = cu_q != nullptr;
  const bool adaptive = (mode & LAMP_ROUTE_ADAPTIVE) != 0;
  const bool skip = !std::isinf(skip_tau) || skip_tau < 0.0f;
  int bm, bn;
  tile_shape(D, &bm, &bn);
  lamp::AttnParams& p = call->p;
  std::memset(&p, 0, sizeof(p));
  const int BHq = B * H, BHk = B * Hkv;
  // TMA views [planes][rows][D]: dense (B*H planes of L rows) or packed (H planes of total rows)
  const int qr = varlen ? total_q : Lq, kr = varlen ? total_k : Lk;
  const int qpl = varlen ? H : BHq, kpl = varlen ? Hkv : BHk;
  if ((r = make_map(&p.tm_q16, q, 2, D, qr, qpl, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))) return r;
  if ((r = make_map(&p.tm_k16, k, 2, D, kr, kpl, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B))) return r;
  if (pv8) {
    if ((r = make_map_pitch(&p.tm_v8, v, Lk, v8_pitch(Lk), D, kpl, bn, D,
                            CU_TENSOR_MAP_SWIZZLE_128B)))
      return r;
    p.v_scale = v_scale;
  } else if ((r = make_map(&p.tm_v, v, 2, D, kr, kpl, 64, bn, CU_TENSOR_MAP_SWIZZLE_128B))) {
    return r;
  }
  const CUtensorMapSwizzle sw8 = (D == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const int in8 = (D == 64) ? 64 : 128;
  if ((r = make_map(&p.tm_q8, q8, 1, D, qr, qpl, in8, 128, sw8))) return r;
  if ((r = make_map(&p.tm_k8, k8, 1, D, kr, kpl, in8, bn, sw8))) return r;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  const int nqt = (Lq + bm - 1) / bm, nkt = (Lk + bn - 1) / bn;
  const int gt = adaptive ? 1 : group_tiles;
  const int ng = (nkt + gt - 1) / gt;
  p.mask = adaptive ? nullptr : mask_bits;
  p.mask_words = (ng + 63) / 64;
  p.group_tiles = gt;
  p.o = o;
  p.lse = lse;
  p.route = route_out;
  p.B = B; p.H = H; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk;
  p.q_rows = qr;
  p.k_rows = kr;
  p.cu_q = cu_q;
  p.cu_k = varlen ? cu_k : nullptr;
  p.n_ct = (Lq + 127) / 128;
  p.nqt = nqt;
  p.nkt = nkt;
  p.causal = causal;
  p.window = window;
  const float sc = (scale > 0.0f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  const float log2e = 1.4426950408889634f;
  p.scale_log2 = sc * log2e;
  p.tau_log2 = adaptive ? tau * log2e : 0.0f;
  p.skip_log2 = skip ? skip_tau * log2e : INFINITY;
  p.adaptive = adaptive ? 1 : 0;
  p.e4m3 = (mode & LAMP_FMT_E4M3) ? 1 : 0;
  p.bf16 = (mode & LAMP_IN_BF16) ? 1 : 0;
  p.out_f32 = (mode & LAMP_OUT_INDTYPE) ? 0 : 1;
  p.wait_ns = kWaitUs * 1000ull;
  call->route_bytes = route_out ? static_cast<size_t>(BHq) * nqt * nkt : 0;
  call->grid = BHq * p.n_ct;  // (check_attn bounds it)
  if (pv8) {
    call->kernel = K_CFG128P8;  // (check_attn: D = 128)
  } else if (D == 64) {
    call->kernel = K_CFG64;
  } else if (D == 128 && !p.e4m3 && !skip && (adaptive || p.mask_words <= 2)) {
    // The two-tile kernel keeps two mask words per query tile (128 key groups); wider masks go
    // to the single-tile kernel, which reads any number of words (as does the threshold skip).
    // Persistent CTAs: one per SM (the kernel fills the SM's shared and tensor memory), each
    // walking its share of the work items (query-tile pairs of two heads of one KV group when
    // the group size is even, else pairs of consecutive query tiles of one head).
    const long long items = ((H / Hkv) % 2 == 0) ? static_cast<long long>(B) * (H / 2) * nqt
                                                 : static_cast<long long>(BHq) * ((nqt + 1) / 2);
    int nsm = 0;
    if ((r = sm_count(&nsm))) return r;
    call->kernel = K_PP;
    call->grid = static_cast<int>(std::min<long long>(items, nsm));
  } else {
    call->kernel = (D == 128) ? K_CFG128 : K_CFG256;
  }
  // Chunks of KV planes for the kernels' work order: the largest divisor of B * Hkv whose K16,
  // V and K8 tiles (5 bytes per element) fit in 40 MB of L2 (one plane at least), so that the
  // work in flight streams one chunk's keys from L2 while Q and O pass through it.  A sliding
  // window already keeps the CTAs of one query tile on one band of keys, and a
  // variable-length batch has its own lengths: one chunk there.  The two-tile kernel, whose
  // persistent CTAs take items in turn, uses the chunked order (with items from a ticket
  // counter, which keeps its CTAs' work even across the chunks) only when all KV planes
  // together exceed L2 (more than 100 MB); below that every key stays in L2 anyway, and the
  // fixed snake order over the longest-first items measured faster (no atomics on the
  // producer's path).
  const int nkv = BHk;
  const double plane = 5.0 * static_cast<double>(Lk) * D;
  p.chunk_kv = nkv;
  call->pp_dynamic = false;
  if (window == 0 && !varlen) {
    for (int d = nkv; d >= 1; --d)
      if (nkv % d == 0 && (d == 1 || d * plane <= 40e6)) {
        p.chunk_kv = d;
        break;
      }
    if (call->kernel == K_PP) {
      call->pp_dynamic = nkv * plane > 100e6;
      if (!call->pp_dynamic) p.chunk_kv = nkv;
    }
  }
  return LAMP_OK;
}

int launch_attn(const AttnCall& c, cudaStream_t st) {
  if (c.route_bytes)
    LAMP_CUDA(cudaMemsetAsync(c.p.route, 0, c.route_bytes, st), "memset route");
  switch (c.kernel) {
    case K_CFG64: return launch_attn_cfg<Cfg64>(c.p, c.grid, st);
    case K_PP: return launch_attn_pp(c.p, c.grid, c.pp_dynamic, st);
    case K_CFG128: return launch_attn_cfg<Cfg128>(c.p, c.grid, st);
    case K_CFG128P8: return launch_attn_pv8(c.p, c.grid, st);
    default: return launch_attn_cfg<Cfg256>(c.p, c.grid, st);
  }
}

// The routed attention kernel on already-quantised operands: checks, then prepare, then launch.
int attn_q8(const void* q, const void* k, const void* v, const void* q8, const void* k8,
            const float* q_scale, const float* k_scale, void* o, float* lse, int B, int H,
            int Hkv, int Lq, int Lk, int D, int causal, int window, float scale,
            const uint64_t* mask_bits, int group_tiles, int mode, float tau, uint8_t* route_out,
            cudaStream_t st, const int* cu_q = nullptr, const int* cu_k = nullptr,
            int total_q = 0, int total_k = 0, float skip_tau = INFINITY) {
  int r = check_attn(q, k, v, true, q8, k8, q_scale, k_scale, o, B, H, Hkv, Lq, Lk, D, causal,
                     window, scale, group_tiles, mode, tau, cu_q, cu_k, total_q, total_k,
                     skip_tau);
  if (r) return r;
  AttnCall call;
  if ((r = prepare_attn(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                        window, scale, mask_bits, group_tiles, mode, tau, route_out, cu_q, cu_k,
                        total_q, total_k, skip_tau, &call)))
    return r;
  return launch_attn(call, st);
}

// Quantise Q and K into `ws` (laid out as w), then run the routed attention: the end-to-end
// path shared by lamp_attn_fwd, lamp_attn_fwd_noalloc and lamp_attn_fwd_varlen.  The caller has
// run check_attn; the tensor maps are built before the quantiser is enqueued, so that a failure
// there leaves the device untouched too.
int quant_and_attend(const void* q, const void* k, const void* v, void* o, float* lse,
                     void* ws, const WsLayout& w, int B, int H, int Hkv, int Lq, int Lk, int D,
                     int causal, int window, float scale, const uint64_t* mask_bits,
                     int group_tiles, int mode, float tau, cudaStream_t st,
                     const int* cu_q = nullptr, const int* cu_k = nullptr, int total_q = 0,
                     int total_k = 0) {
  auto* base = static_cast<uint8_t*>(ws);
  uint8_t* q8 = base + w.q8;
  uint8_t* k8 = base + w.k8;
  float* qs = reinterpret_cast<float*>(base + w.qs);
  float* ks = reinterpret_cast<float*>(base + w.ks);
  const bool pv8 = (mode & LAMP_PV_E4M3) != 0;  // (dense batches only: check_attn)
  uint8_t* v8 = base + w.v8;
  float* vs = reinterpret_cast<float*>(base + w.vs);
  AttnCall call;
  int r = prepare_attn(q, k, pv8 ? static_cast<const void*>(v8) : v, q8, k8, qs, ks, o, lse, B, H,
                       Hkv, Lq, Lk, D, causal, window, scale, mask_bits, group_tiles, mode, tau,
                       nullptr, cu_q, cu_k, total_q, total_k, INFINITY, &call,
                       pv8 ? vs : nullptr);
  if (r) return r;
  if ((r = quant_qk(q, k, q8, k8, qs, ks, B, H, Hkv, Lq, Lk, D, mode, st, cu_q, cu_k, total_q,
                    total_k)))
    return r;
  if (pv8 && (r = quant_v(v, v8, vs, B, Hkv, Lk, D, mode, st))) return r;
  return launch_attn(call, st);
}

}  // namespace

namespace {
template <int KIND, int N>
int probe_launch(int nsm, int iters, cudaStream_t st) {
  static bool attr_set[64] = {};
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_UNSUPPORTED, "device index %d", dev);
  if (!attr_set[dev]) {
    LAMP_CUDA(cudaFuncSetAttribute(lamp::mma_probe_kernel<KIND, N>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, lamp::PROBE_SMEM),
              "cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  lamp::mma_probe_kernel<KIND, N><<<nsm, lamp::PROBE_THREADS, lamp::PROBE_SMEM, st>>>(iters, kWaitUs);
  LAMP_CUDA(cudaGetLastError(), "mma_probe_kernel launch");
  return LAMP_OK;
}

template <int KIND>
int probe_n(int n, int nsm, int iters, cudaStream_t st) {
  if (n == 64) return probe_launch<KIND, 64>(nsm, iters, st);
  if (n == 128) return probe_launch<KIND, 128>(nsm, iters, st);
  return probe_launch<KIND, 256>(nsm, iters, st);
}

// ---- structured static routing template, host side -------------------------------------

// Group of the diagonal key tile of routing row qt: the tile of the key aligned with the
// row's last query (bottom-right), clamped to the key range.
long long template_gd(int qt, int bm, int bn, int Lq, int Lk, int nkt, int group_tiles) {
  const long long aligned = static_cast<long long>(std::min(Lq, (qt + 1) * bm)) - 1 + Lk - Lq;
  const long long kd = aligned < 0 ? 0 : std::min<long long>(aligned / bn, nkt - 1);
  return kd / group_tiles;
}

struct TemplateGeo {
  int bm, bn, nqt, nkt, ng;
  std::vector<long long> pairs;  // visible pairs of one (batch, head) per (qt, group)
  long long total;
};

// Visible pairs per (routing row, key group) under the causal / window limits of the kernel.
int template_geo(int Lq, int Lk, int D, int group_tiles, int causal, int window,
                 TemplateGeo* t) {
  if (Lq < 1 || Lk < 1 || group_tiles < 1 || window < 0 || Lq > (1 << 30) || Lk > (1 << 30))
    return fail(LAMP_ERR_INVALID, "invalid template geometry");
  if (window > 0 && !causal) return fail(LAMP_ERR_UNSUPPORTED, "window needs causal = 1");
  if (tile_shape(D, &t->bm, &t->bn) != LAMP_OK)
    return fail(LAMP_ERR_UNSUPPORTED, "head dimension D=%d not supported (64, 128, 256)", D);
  t->nqt = (Lq + t->bm - 1) / t->bm;
  t->nkt = (Lk + t->bn - 1) / t->bn;
  t->ng = (t->nkt + group_tiles - 1) / group_tiles;
  t->pairs.assign(static_cast<size_t>(t->nqt) * t->ng, 0);
  t->total = 0;
  const long long gk = static_cast<long long>(group_tiles) * t->bn;  // keys per group
  for (int i = 0; i < Lq; ++i) {
    long long lo = 0, hi = Lk - 1;
    if (causal) {
      hi = std::min<long long>(static_cast<long long>(i) + Lk - Lq, Lk - 1);
      if (window > 0) lo = std::max<long long>(0, static_cast<long long>(i) + Lk - Lq - window + 1);
    }
    if (hi < lo) continue;
    long long* row = t->pairs.data() + static_cast<size_t>(i / t->bm) * t->ng;
    for (long long g = lo / gk; g <= hi / gk; ++g) {
      const long long a = std::max(lo, g * gk), b = std::min(hi, (g + 1) * gk - 1);
      row[g] += b - a + 1;
      t->total += b - a + 1;
    }
  }
  return LAMP_OK;
}

bool template_sixteen(long long g, long long gd, int sink, int band, int stride) {
  const long long d = gd >= g ? gd - g : g - gd;
  return g < sink || d < band || (stride > 0 && d % stride == 0);
}
}  // namespace

namespace {
template <int D, bool E4M3, int GM>
int launch_decode_t(const lamp::DecodeParams& p, cudaStream_t st) {
  constexpr int smem = lamp::DecSmem<D>::BYTES;
  static bool attr_set[64] = {};
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    LAMP_CUDA(cudaFuncSetAttribute(lamp::decode_split_kernel<D, E4M3, GM>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
              "cudaFuncSetAttribute");
    attr_set[dev] = true;
  }
  const dim3 grid(p.nsplit, p.B * p.Hkv);
  lamp::decode_split_kernel<D, E4M3, GM><<<grid, lamp::dec_threads(D), smem, st>>>(p);
  LAMP_CUDA(cudaGetLastError(), "decode_split_kernel launch");
  lamp::decode_combine_kernel<D><<<p.B * p.H, lamp::DEC_COMBINE_THREADS,
                                   (p.nsplit + 64) * sizeof(float), st>>>(p);
  LAMP_CUDA(cudaGetLastError(), "decode_combine_kernel launch");
  return LAMP_OK;
}

// per-head loops bounded by the group size rounded up to a power of two
template <int D, bool E4M3>
int launch_decode_g(const lamp::DecodeParams& p, cudaStream_t st) {
  if (p.G <= 1) return launch_decode_t<D, E4M3, 1>(p, st);
  if (p.G <= 2) return launch_decode_t<D, E4M3, 2>(p, st);
  if (p.G <= 4) return launch_decode_t<D, E4M3, 4>(p, st);
  return launch_decode_t<D, E4M3, 8>(p, st);
}

template <int D>
int launch_decode(const lamp::DecodeParams& p, cudaStream_t st) {
  return p.e4m3 ? launch_decode_g<D, true>(p, st) : launch_decode_g<D, false>(p, st);
}
}  // namespace

extern "C" {

int lamp_tile_shape(int D, int* bm, int* bn) {
  if (!bm || !bn) return fail(LAMP_ERR_INVALID, "null output pointer");
  int r = tile_shape(D, bm, bn);
  if (r) return fail(r, "head dimension D=%d not supported (64, 128, 256)", D);
  return LAMP_OK;
}

int lamp_mask_words(int Lk, int D, int group_tiles) {
  int bm, bn;
  if (Lk < 1 || group_tiles < 1 || tile_shape(D, &bm, &bn) != LAMP_OK) return -1;
  const int nkt = (Lk + bn - 1) / bn;
  const int ng = (nkt + group_tiles - 1) / group_tiles;
  return (ng + 63) / 64;
}

int lamp_quant_qk(const void* q, const void* k, void* q8, void* k8, float* q_scale,
                  float* k_scale, int B, int H, int Hkv, int Lq, int Lk, int D, int mode,
                  void* stream) {
  int r = check_sizes(B, H, Hkv, Lq, Lk, D);
  if (r) return r;
  if ((q == nullptr) != (q8 == nullptr) || (q == nullptr) != (q_scale == nullptr))
    return fail(LAMP_ERR_INVALID, "q, q8 and q_scale must be all set or all null");
  if ((k == nullptr) != (k8 == nullptr) || (k == nullptr) != (k_scale == nullptr))
    return fail(LAMP_ERR_INVALID, "k, k8 and k_scale must be all set or all null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8))
    return fail(LAMP_ERR_INVALID, "q, k, q8, k8 must be 16-byte aligned");
  return quant_qk(q, k, q8, k8, q_scale, k_scale, B, H, Hkv, Lq, Lk, D, mode,
                  static_cast<cudaStream_t>(stream));
}

int lamp_build_mask(uint64_t* mask_bits, int B, int H, int Lq, int Lk, int D, int group_tiles,
                    float fp16_fraction, uint64_t seed, void* stream) {
  if (!mask_bits) return fail(LAMP_ERR_INVALID, "null mask pointer");
  int r = check_sizes(B, H, 1, Lq, Lk, D);
  if (r) return r;
  if (group_tiles < 1) return fail(LAMP_ERR_INVALID, "group_tiles must be >= 1");
  if (!(fp16_fraction >= 0.0f && fp16_fraction <= 1.0f))
    return fail(LAMP_ERR_INVALID, "fp16_fraction must be in [0, 1]");
  int bm, bn;
  tile_shape(D, &bm, &bn);
  const int nqt = (Lq + bm - 1) / bm, nkt = (Lk + bn - 1) / bn;
  const int ng = (nkt + group_tiles - 1) / group_tiles;
  const int W = (ng + 63) / 64;
  const long long rows = static_cast<long long>(B) * H * nqt;
  const long long total = rows * W;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 148 * 16);
  lamp::mask_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      mask_bits, rows, ng, W, static_cast<double>(fp16_fraction), seed);
  LAMP_CUDA(cudaGetLastError(), "mask_kernel launch");
  return LAMP_OK;
}

int lamp_build_mask_template(uint64_t* mask_bits, int B, int H, int Lq, int Lk, int D,
                             int group_tiles, int sink_groups, int band_groups,
                             int stride_groups, void* stream) {
  if (!mask_bits) return fail(LAMP_ERR_INVALID, "null mask pointer");
  int r = check_sizes(B, H, 1, Lq, Lk, D);
  if (r) return r;
  if (group_tiles < 1) return fail(LAMP_ERR_INVALID, "group_tiles must be >= 1");
  if (sink_groups < 0 || band_groups < 0 || stride_groups < 0)
    return fail(LAMP_ERR_INVALID, "template parameters must be >= 0");
  int bm, bn;
  tile_shape(D, &bm, &bn);
  const int nqt = (Lq + bm - 1) / bm, nkt = (Lk + bn - 1) / bn;
  const int ng = (nkt + group_tiles - 1) / group_tiles;
  const int W = (ng + 63) / 64;
  const long long rows = static_cast<long long>(B) * H * nqt;
  const long long total = rows * W;
  const int threads = 256;
  const long long blocks = std::min<long long>((total + threads - 1) / threads, 148 * 16);
  lamp::mask_template_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                               static_cast<cudaStream_t>(stream)>>>(
      mask_bits, rows, nqt, ng, W, Lq, Lk, bm, bn, nkt, group_tiles, sink_groups, band_groups,
      stride_groups);
  LAMP_CUDA(cudaGetLastError(), "mask_template_kernel launch");
  return LAMP_OK;
}

int lamp_template_fraction(int Lq, int Lk, int D, int group_tiles, int causal, int window,
                           int sink_groups, int band_groups, int stride_groups,
                           double* fp16_fraction) {
  if (!fp16_fraction) return fail(LAMP_ERR_INVALID, "null output pointer");
  if (sink_groups < 0 || band_groups < 0 || stride_groups < 0)
    return fail(LAMP_ERR_INVALID, "template parameters must be >= 0");
  TemplateGeo t;
  int r = template_geo(Lq, Lk, D, group_tiles, causal, window, &t);
  if (r) return r;
  long long sixteen = 0;
  for (int qt = 0; qt < t.nqt; ++qt) {
    const long long gd = template_gd(qt, t.bm, t.bn, Lq, Lk, t.nkt, group_tiles);
    for (int g = 0; g < t.ng; ++g)
      if (template_sixteen(g, gd, sink_groups, band_groups, stride_groups))
        sixteen += t.pairs[static_cast<size_t>(qt) * t.ng + g];
  }
  *fp16_fraction = t.total ? static_cast<double>(sixteen) / static_cast<double>(t.total) : 0.0;
  return LAMP_OK;
}

int lamp_template_for_int8_fraction(int Lq, int Lk, int D, int group_tiles, int causal,
                                    int window, double int8_fraction, int* sink_groups,
                                    int* band_groups, int* stride_groups,
                                    double* fp16_fraction) {
  if (!sink_groups || !band_groups || !stride_groups || !fp16_fraction)
    return fail(LAMP_ERR_INVALID, "null output pointer");
  if (!(int8_fraction >= 0.0 && int8_fraction <= 1.0))
    return fail(LAMP_ERR_INVALID, "int8_fraction must be in [0, 1]");
  TemplateGeo t;
  int r = template_geo(Lq, Lk, D, group_tiles, causal, window, &t);
  if (r) return r;
  // visible pairs by distance |gd - g| from the diagonal group, split into group 0 (the sink
  // candidate) and the rest: every candidate is then scored in O(nG)
  std::vector<long long> h0(t.ng, 0), hr(t.ng, 0);
  for (int qt = 0; qt < t.nqt; ++qt) {
    const long long gd = template_gd(qt, t.bm, t.bn, Lq, Lk, t.nkt, group_tiles);
    for (int g = 0; g < t.ng; ++g) {
      const long long d = gd >= g ? gd - g : g - gd;
      (g == 0 ? h0 : hr)[d] += t.pairs[static_cast<size_t>(qt) * t.ng + g];
    }
  }
  long long sink_pairs = 0;
  for (int d = 0; d < t.ng; ++d) sink_pairs += h0[d];
  const double target = 1.0 - int8_fraction;
  double best_err = 2.0, best_frac = 0.0;
  int best[3] = {0, 0, 0};
  const int sinks[2] = {1, 0};
  for (int si = 0; si < 2; ++si) {
    const int sink = sinks[si];
    for (int stride = 0; stride <= t.ng; stride = (stride == 0) ? 2 : stride + 1) {
      for (int band = 1; band <= t.ng; ++band) {
        long long sixteen = sink ? sink_pairs : 0;
        for (int d = 0; d < t.ng; ++d) {
          const bool sel = d < band || (stride > 0 && d % stride == 0);
          if (sel) sixteen += hr[d] + (sink ? 0 : h0[d]);
        }
        const double frac = t.total ? static_cast<double>(sixteen) / t.total : 0.0;
        const double err = std::fabs(frac - target);
        if (err < best_err - 1e-12) {
          best_err = err;
          best_frac = frac;
          best[0] = sink;
          best[1] = band;
          best[2] = stride;
        }
      }
    }
  }
  *sink_groups = best[0];
  *band_groups = best[1];
  *stride_groups = best[2];
  *fp16_fraction = best_frac;
  return LAMP_OK;
}

int lamp_attn_fwd_q8(const void* q, const void* k, const void* v, const void* q8,
                     const void* k8, const float* q_scale, const float* k_scale, void* o,
                     float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                     int window, float scale, const uint64_t* mask_bits, int group_tiles,
                     int mode, float tau, uint8_t* route_out, void* stream) {
  if ((mode & ~0x1Fu) == 0 && (mode & LAMP_PV_E4M3))  // (unknown bits: check_attn's error)
    return fail(LAMP_ERR_UNSUPPORTED, "8-bit P.V takes the 8-bit V: lamp_attn_fwd_q8_pv8");
  return attn_q8(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                 window, scale, mask_bits, group_tiles, mode, tau, route_out,
                 static_cast<cudaStream_t>(stream));
}

int lamp_attn_fwd_q8_pv8(const void* q, const void* k, const void* q8, const void* k8,
                         const float* q_scale, const float* k_scale, const void* v8t,
                         const float* v_scale, void* o, float* lse, int B, int H, int Hkv,
                         int Lq, int Lk, int D, int causal, int window, float scale,
                         const uint64_t* mask_bits, int group_tiles, int mode, float tau,
                         void* stream) {
  if (!(mode & LAMP_PV_E4M3)) return fail(LAMP_ERR_INVALID, "mode must include LAMP_PV_E4M3");
  if (!v_scale) return fail(LAMP_ERR_INVALID, "null v_scale");
  int r = check_attn(q, k, v8t, true, q8, k8, q_scale, k_scale, o, B, H, Hkv, Lq, Lk, D, causal,
                     window, scale, group_tiles, mode, tau, nullptr, nullptr, 0, 0, INFINITY);
  if (r) return r;
  AttnCall call;
  if ((r = prepare_attn(q, k, v8t, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D,
                        causal, window, scale, mask_bits, group_tiles, mode, tau, nullptr,
                        nullptr, nullptr, 0, 0, INFINITY, &call, v_scale)))
    return r;
  return launch_attn(call, static_cast<cudaStream_t>(stream));
}

int lamp_quant_v(const void* v, void* v8t, float* v_scale, int B, int Hkv, int Lk, int D,
                 int mode, void* stream) {
  int r = check_sizes(B, Hkv, Hkv, 1, Lk, D);
  if (r) return r;
  if (!v || !v8t || !v_scale) return fail(LAMP_ERR_INVALID, "null pointer");
  if (!aligned16(v8t)) return fail(LAMP_ERR_INVALID, "v8t must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(v) & 1u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    return fail(LAMP_ERR_INVALID, "v and v_scale must be aligned to their elements");
  return quant_v(v, v8t, v_scale, B, Hkv, Lk, D, mode, static_cast<cudaStream_t>(stream));
}

int lamp_attn_debug(const void* q, const void* k, const void* v, const void* q8,
                    const void* k8, const float* q_scale, const float* k_scale, void* o,
                    float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                    int window, float scale, const uint64_t* mask_bits, int group_tiles,
                    int mode, float tau, uint8_t* route_out, const int* tile_slot, int n_slots,
                    void* s8_dump, void* s16_dump, void* stream) {
  if ((mode & ~0x1Fu) == 0 && (mode & LAMP_PV_E4M3))
    return fail(LAMP_ERR_UNSUPPORTED, "no debug capture of the 8-bit P.V mode");
  if (!tile_slot || n_slots < 1) return fail(LAMP_ERR_INVALID, "a slot map and n_slots >= 1 are needed");
  if (!s8_dump && !s16_dump) return fail(LAMP_ERR_INVALID, "no dump buffer");
  if (!aligned16(s8_dump) || !aligned16(s16_dump))
    return fail(LAMP_ERR_INVALID, "dump buffers must be 16-byte aligned");
  int r = check_attn(q, k, v, true, q8, k8, q_scale, k_scale, o, B, H, Hkv, Lq, Lk, D, causal,
                     window, scale, group_tiles, mode, tau, nullptr, nullptr, 0, 0, INFINITY);
  if (r) return r;
  AttnCall call;
  if ((r = prepare_attn(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal,
                        window, scale, mask_bits, group_tiles, mode, tau, route_out, nullptr,
                        nullptr, 0, 0, INFINITY, &call)))
    return r;
  call.p.dbg_slot = tile_slot;
  call.p.dbg_s8 = static_cast<uint32_t*>(s8_dump);
  call.p.dbg_s16 = static_cast<uint32_t*>(s16_dump);
  call.p.dbg_nslots = n_slots;
  return launch_attn(call, static_cast<cudaStream_t>(stream));
}

int lamp_exp2_eval(const float* x, float* y, int n, int method, void* stream) {
  if (!x || !y || n < 0) return fail(LAMP_ERR_INVALID, "null pointer or negative n");
  if (method != 0 && method != 1) return fail(LAMP_ERR_INVALID, "method must be 0 or 1");
  if (n == 0) return LAMP_OK;
  const int pairs = (n + 1) / 2;
  const int grid = std::min((pairs + 255) / 256, 148 * 8);
  lamp::exp2_eval_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, method);
  LAMP_CUDA(cudaGetLastError(), "exp2_eval_kernel launch");
  return LAMP_OK;
}

size_t lamp_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int D, int mode) {
  int bm, bn;
  if (B < 1 || H < 1 || Hkv < 1 || Lq < 1 || Lk < 1 || tile_shape(D, &bm, &bn) != LAMP_OK)
    return 0;
  return ws_layout(B, H, Hkv, Lq, Lk, D, 0, 0, (mode & LAMP_PV_E4M3) != 0).total;
}

int lamp_set_workspace(void* ptr, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 255u))
    return fail(LAMP_ERR_INVALID, "workspace must be 256-byte aligned");
  g_ws.user = ptr;
  g_ws.user_bytes = ptr ? bytes : 0;
  return LAMP_OK;
}

int lamp_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int Hkv, int Lq, int Lk, int D, int causal, int window, float scale,
                  const uint64_t* mask_bits, int group_tiles, int mode, float tau, void* stream) {
  int r = check_attn(q, k, v, false, nullptr, nullptr, nullptr, nullptr, o, B, H, Hkv, Lq, Lk,
                     D, causal, window, scale, group_tiles, mode, tau, nullptr, nullptr, 0, 0,
                     INFINITY);
  if (r) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(B, H, Hkv, Lq, Lk, D, 0, 0, (mode & LAMP_PV_E4M3) != 0);
  void* ws = nullptr;
  if ((r = get_workspace(w.total, st, &ws))) return r;
  return quant_and_attend(q, k, v, o, lse, ws, w, B, H, Hkv, Lq, Lk, D, causal, window, scale,
                          mask_bits, group_tiles, mode, tau, st);
}

namespace {
// Per-device resources of lamp_attn_fwd_host: a host-to-device and a device-to-host copy stream
// and the events of two buffer slots, created on first use and kept for the process.
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t fork = nullptr, join_in = nullptr, join_out = nullptr;
  cudaEvent_t in_done[2] = {}, cmp_done[2] = {}, out_done[2] = {};
};
HostPipe g_pipe[64];
std::mutex g_pipe_mu;

int host_pipe(HostPipe** out) {
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_INVALID, "device index out of range");
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    LAMP_CUDA(cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking), "cudaStreamCreate(in)");
    LAMP_CUDA(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking), "cudaStreamCreate(out)");
    cudaEvent_t* evs[] = {&hp.fork, &hp.join_in, &hp.join_out, &hp.in_done[0], &hp.in_done[1],
                          &hp.cmp_done[0], &hp.cmp_done[1], &hp.out_done[0], &hp.out_done[1]};
    for (cudaEvent_t* e : evs)
      LAMP_CUDA(cudaEventCreateWithFlags(e, cudaEventDisableTiming), "cudaEventCreate");
    hp.ready = true;
  }
  *out = &hp;
  return LAMP_OK;
}
}  // namespace

int lamp_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int Hkv, int Lq, int Lk, int D, int causal, int window,
                       float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                       float tau, int n_chunks, void* stream) {
  if (!q || !k || !v || !o) return fail(LAMP_ERR_INVALID, "null operand pointer");
  if (n_chunks < 0) return fail(LAMP_ERR_INVALID, "n_chunks must be >= 0");
  // The host buffers need no alignment: the kernels' operands are the device chunks.  Every
  // other check of lamp_attn_fwd runs here, on stand-in aligned addresses.
  alignas(256) static const char kStandIn[256] = {};
  int r = check_attn(kStandIn, kStandIn, kStandIn, false, nullptr, nullptr, nullptr, nullptr,
                     kStandIn, B, H, Hkv, Lq, Lk, D, causal, window, scale, group_tiles, mode,
                     tau, nullptr, nullptr, 0, 0, INFINITY);
  if (r) return r;
  const int G = H / Hkv;
  const int planes = B * Hkv;  // (b, kvh): G query heads and one KV head, an independent problem
  const size_t eb = 2, ob = (mode & LAMP_OUT_INDTYPE) ? 2 : 4;
  const size_t q_pl = static_cast<size_t>(G) * Lq * D * eb;   // bytes of one plane's Q
  const size_t kv_pl = static_cast<size_t>(Lk) * D * eb;      // ... of its K (and of its V)
  const size_t o_pl = static_cast<size_t>(G) * Lq * D * ob;   // ... of its O
  const size_t l_pl = static_cast<size_t>(G) * Lq * sizeof(float);
  if (n_chunks == 0) {  // about 256 MB of copies per chunk, at most 8 chunks
    const double bytes = static_cast<double>(planes) * (q_pl + 2 * kv_pl + o_pl + l_pl);
    n_chunks = static_cast<int>(std::max(1.0, std::min(8.0, std::floor(bytes / 256e6))));
  }
  n_chunks = std::min(n_chunks, planes);
  const int per = (planes + n_chunks - 1) / n_chunks;  // planes per chunk (the last may be short)
  n_chunks = (planes + per - 1) / per;
  // workspace: the quantiser's codes and scales for one chunk, then two slots of device chunks
  const WsLayout wq = ws_layout(per, G, 1, Lq, Lk, D, 0, 0, (mode & LAMP_PV_E4M3) != 0);
  const size_t s_q = 0, s_k = align256(per * q_pl), s_v = s_k + align256(per * kv_pl),
               s_o = s_v + align256(per * kv_pl), s_l = s_o + align256(per * o_pl),
               slot = s_l + align256(per * l_pl);
  const size_t need = align256(wq.total) + 2 * slot;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lk(g_pipe_mu);
  HostPipe* hp = nullptr;
  if ((r = host_pipe(&hp))) return r;
  void* ws = nullptr;
  if ((r = get_workspace(need, st, &ws))) return r;
  auto* base = static_cast<uint8_t*>(ws);
  uint8_t* slots = base + align256(wq.total);
  int bm = 0, bn = 0;
  tile_shape(D, &bm, &bn);
  const size_t mask_pl = mask_bits ? static_cast<size_t>(G) * ((Lq + bm - 1) / bm) *
                                         lamp_mask_words(Lk, D, group_tiles)
                                   : 0;  // mask words of one plane
  const auto* hq = static_cast<const uint8_t*>(q);
  const auto* hk = static_cast<const uint8_t*>(k);
  const auto* hv = static_cast<const uint8_t*>(v);
  auto* ho = static_cast<uint8_t*>(o);
  auto* hl = reinterpret_cast<uint8_t*>(lse);
  // fork: the copy streams start behind the work already queued on `stream`
  LAMP_CUDA(cudaEventRecord(hp->fork, st), "cudaEventRecord");
  LAMP_CUDA(cudaStreamWaitEvent(hp->in, hp->fork, 0), "cudaStreamWaitEvent");
  LAMP_CUDA(cudaStreamWaitEvent(hp->out, hp->fork, 0), "cudaStreamWaitEvent");
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    const int p0 = c * per, np = std::min(per, planes - p0);
    uint8_t* d = slots + s * slot;
    // in: chunk c's Q, K, V, once chunk c - 2 (same slot) has been computed
    if (c >= 2) LAMP_CUDA(cudaStreamWaitEvent(hp->in, hp->cmp_done[s], 0), "cudaStreamWaitEvent");
    LAMP_CUDA(cudaMemcpyAsync(d + s_q, hq + p0 * q_pl, np * q_pl, cudaMemcpyHostToDevice, hp->in),
              "copy Q to the device");
    LAMP_CUDA(cudaMemcpyAsync(d + s_k, hk + p0 * kv_pl, np * kv_pl, cudaMemcpyHostToDevice, hp->in),
              "copy K to the device");
    LAMP_CUDA(cudaMemcpyAsync(d + s_v, hv + p0 * kv_pl, np * kv_pl, cudaMemcpyHostToDevice, hp->in),
              "copy V to the device");
    LAMP_CUDA(cudaEventRecord(hp->in_done[s], hp->in), "cudaEventRecord");
    // compute on `stream`: chunk c as B = np problems of G query heads and one KV head, once
    // its inputs are in and chunk c - 2's outputs have been copied out
    LAMP_CUDA(cudaStreamWaitEvent(st, hp->in_done[s], 0), "cudaStreamWaitEvent");
    if (c >= 2) LAMP_CUDA(cudaStreamWaitEvent(st, hp->out_done[s], 0), "cudaStreamWaitEvent");
    if ((r = quant_and_attend(d + s_q, d + s_k, d + s_v, d + s_o,
                              lse ? reinterpret_cast<float*>(d + s_l) : nullptr, base, wq, np, G,
                              1, Lq, Lk, D, causal, window, scale,
                              mask_bits ? mask_bits + p0 * mask_pl : nullptr, group_tiles, mode,
                              tau, st)))
      return r;
    LAMP_CUDA(cudaEventRecord(hp->cmp_done[s], st), "cudaEventRecord");
    // out: chunk c's O and lse
    LAMP_CUDA(cudaStreamWaitEvent(hp->out, hp->cmp_done[s], 0), "cudaStreamWaitEvent");
    LAMP_CUDA(cudaMemcpyAsync(ho + p0 * o_pl, d + s_o, np * o_pl, cudaMemcpyDeviceToHost, hp->out),
              "copy O to the host");
    if (lse)
      LAMP_CUDA(cudaMemcpyAsync(hl + p0 * l_pl, d + s_l, np * l_pl, cudaMemcpyDeviceToHost,
                                hp->out),
                "copy lse to the host");
    LAMP_CUDA(cudaEventRecord(hp->out_done[s], hp->out), "cudaEventRecord");
  }
  // join: `stream` continues once every copy has completed
  LAMP_CUDA(cudaEventRecord(hp->join_in, hp->in), "cudaEventRecord");
  LAMP_CUDA(cudaEventRecord(hp->join_out, hp->out), "cudaEventRecord");
  LAMP_CUDA(cudaStreamWaitEvent(st, hp->join_in, 0), "cudaStreamWaitEvent");
  LAMP_CUDA(cudaStreamWaitEvent(st, hp->join_out, 0), "cudaStreamWaitEvent");
  return LAMP_OK;
}

int lamp_attn_fwd_q8_skip(const void* q, const void* k, const void* v, const void* q8,
                          const void* k8, const float* q_scale, const float* k_scale, void* o,
                          float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                          int window, float scale, int mode, float tau, float skip_tau,
                          uint8_t* route_out, void* stream) {
  if (!(mode & LAMP_ROUTE_ADAPTIVE)) return fail(LAMP_ERR_INVALID, "the skip needs look-ahead mode");
  if (!(skip_tau == skip_tau)) return fail(LAMP_ERR_INVALID, "skip_tau is NaN");
  return attn_q8(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, Lq, Lk, D, causal, window,
                 scale, nullptr, 1, mode, tau, route_out, static_cast<cudaStream_t>(stream),
                 nullptr, nullptr, 0, 0, skip_tau);
}


int lamp_decode_fwd(const void* q, const void* q8, const float* q_scale, const void* k8,
                    const float* k_scale, const void* v8, const float* v_scale, const int* len_k,
                    float* o, float* lse, int B, int H, int Hkv, int max_k, int D, float scale,
                    const uint64_t* mask_bits, int group_tiles, int mode, void* stream) {
  int r = check_sizes(B, H, Hkv, 1, max_k, D);
  if (r) return r;
  if (!q || !q8 || !q_scale || !k8 || !k_scale || !v8 || !v_scale || !o || !lse)
    return fail(LAMP_ERR_INVALID, "null pointer");
  if (!aligned16(k8) || !aligned16(v8) || !aligned16(q8) || !aligned16(q))
    return fail(LAMP_ERR_INVALID, "q, q8, k8, v8 must be 16-byte aligned");
  if ((mode & ~0x7u) != 0 || (mode & LAMP_ROUTE_ADAPTIVE))
    return fail(LAMP_ERR_UNSUPPORTED, "decode takes bitmask routing and fp32 output only");
  if (H / Hkv > lamp::DEC_MAX_G)
    return fail(LAMP_ERR_UNSUPPORTED, "more than %d query heads per KV head", lamp::DEC_MAX_G);
  if (mask_bits && group_tiles < 1) return fail(LAMP_ERR_INVALID, "group_tiles must be >= 1");
  if (!(scale == scale)) return fail(LAMP_ERR_INVALID, "scale is NaN");
  int bm, bn;
  tile_shape(D, &bm, &bn);
  lamp::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const uint16_t*>(q);
  p.q8 = static_cast<const uint8_t*>(q8);
  p.q_scale = q_scale;
  p.k8 = static_cast<const uint8_t*>(k8);
  p.k_scale = k_scale;
  p.v8 = static_cast<const uint8_t*>(v8);
  p.v_scale = v_scale;
  p.len_k = len_k;
  p.mask = mask_bits;
  p.o = o;
  p.lse = lse;
  p.B = B; p.H = H; p.Hkv = Hkv; p.G = H / Hkv; p.max_k = max_k;
  p.bn = bn;
  p.nkt = (max_k + bn - 1) / bn;
  const int nchunk = (max_k + lamp::DEC_CHUNK - 1) / lamp::DEC_CHUNK;
  p.nsplit = (nchunk + lamp::DEC_SPLIT_CHUNKS - 1) / lamp::DEC_SPLIT_CHUNKS;
  p.wait_us = kWaitUs;
  p.group_tiles = mask_bits ? group_tiles : 1;
  p.mask_words = ((p.nkt + p.group_tiles - 1) / p.group_tiles + 63) / 64;
  p.scale = (scale > 0.0f) ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.e4m3 = (mode & LAMP_FMT_E4M3) ? 1 : 0;
  p.bf16 = (mode & LAMP_IN_BF16) ? 1 : 0;
  const size_t need = static_cast<size_t>(B) * H * p.nsplit * (2 + D) * sizeof(float);
  void* ws = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((r = get_workspace(need, st, &ws))) return r;
  p.part = static_cast<float*>(ws);
  if (D == 64) return launch_decode<64>(p, st);
  if (D == 128) return launch_decode<128>(p, st);
  return launch_decode<256>(p, st);
}

int lamp_quant_qk_varlen(const void* q, const void* k, void* q8, void* k8, float* q_scale,
                         float* k_scale, const int* cu_q, const int* cu_k, int B, int H,
                         int Hkv, int max_q, int max_k, int total_q, int total_k, int D,
                         int mode, void* stream) {
  int r = check_sizes(B, H, Hkv, max_q, max_k, D);
  if (r) return r;
  if ((q == nullptr) != (q8 == nullptr) || (q == nullptr) != (q_scale == nullptr) ||
      (q != nullptr && (cu_q == nullptr || total_q < 1 || total_q > (1 << 30))))
    return fail(LAMP_ERR_INVALID, "q, q8, q_scale, cu_q must be all set (total_q > 0) or q null");
  if ((k == nullptr) != (k8 == nullptr) || (k == nullptr) != (k_scale == nullptr) ||
      (k != nullptr && (cu_k == nullptr || total_k < 1 || total_k > (1 << 30))))
    return fail(LAMP_ERR_INVALID, "k, k8, k_scale, cu_k must be all set (total_k > 0) or k null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8))
    return fail(LAMP_ERR_INVALID, "q, k, q8, k8 must be 16-byte aligned");
  return quant_qk(q, k, q8, k8, q_scale, k_scale, B, H, Hkv, max_q, max_k, D, mode,
                  static_cast<cudaStream_t>(stream), cu_q, cu_k, total_q, total_k);
}

int lamp_attn_fwd_q8_varlen(const void* q, const void* k, const void* v, const void* q8,
                            const void* k8, const float* q_scale, const float* k_scale,
                            void* o, float* lse, const int* cu_q, const int* cu_k, int B, int H,
                            int Hkv, int max_q, int max_k, int total_q, int total_k, int D,
                            int causal, int window, float scale, const uint64_t* mask_bits,
                            int group_tiles, int mode, float tau, uint8_t* route_out,
                            void* stream) {
  if (!cu_q || !cu_k) return fail(LAMP_ERR_INVALID, "null sequence offsets");
  return attn_q8(q, k, v, q8, k8, q_scale, k_scale, o, lse, B, H, Hkv, max_q, max_k, D, causal,
                 window, scale, mask_bits, group_tiles, mode, tau, route_out,
                 static_cast<cudaStream_t>(stream), cu_q, cu_k, total_q, total_k);
}

int lamp_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int* cu_q, const int* cu_k, int B, int H, int Hkv, int max_q,
                         int max_k, int total_q, int total_k, int D, int causal, int window,
                         float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                         float tau, void* stream) {
  if (!cu_q || !cu_k) return fail(LAMP_ERR_INVALID, "null sequence offsets");
  int r = check_attn(q, k, v, false, nullptr, nullptr, nullptr, nullptr, o, B, H, Hkv, max_q,
                     max_k, D, causal, window, scale, group_tiles, mode, tau, cu_q, cu_k, total_q,
                     total_k, INFINITY);
  if (r) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(B, H, Hkv, max_q, max_k, D, total_q, total_k);
  void* ws = nullptr;
  if ((r = get_workspace(w.total, st, &ws))) return r;
  return quant_and_attend(q, k, v, o, lse, ws, w, B, H, Hkv, max_q, max_k, D, causal, window,
                          scale, mask_bits, group_tiles, mode, tau, st, cu_q, cu_k, total_q,
                          total_k);
}

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_base[64] = {};

// Device address of the scratch array on the current device (looked up once per device).
int noalloc_base(void** out) {
  int dev = 0;
  LAMP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LAMP_ERR_INVALID, "device index out of range");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_base[dev]) {
    void* p = nullptr;
    LAMP_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
    if (!p) return fail(LAMP_ERR_CUDA, "scratch array has no device address");
    g_noalloc_base[dev] = p;
  }
  *out = g_noalloc_base[dev];
  return LAMP_OK;
}
}  // namespace

int lamp_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int Hkv, int Lq, int Lk, int D, int causal, int window,
                          float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                          float tau, void* stream) {
  int r = check_attn(q, k, v, false, nullptr, nullptr, nullptr, nullptr, o, B, H, Hkv, Lq, Lk,
                     D, causal, window, scale, group_tiles, mode, tau, nullptr, nullptr, 0, 0,
                     INFINITY);
  if (r) return r;
  const WsLayout w = ws_layout(B, H, Hkv, Lq, Lk, D, 0, 0, (mode & LAMP_PV_E4M3) != 0);
  if (w.total > static_cast<size_t>(LAMP_NOALLOC_MAX_BYTES))
    return fail(LAMP_ERR_INVALID,
                "problem needs %zu bytes of scratch; lamp_attn_fwd_noalloc holds at most %zu "
                "(use lamp_attn_fwd with a workspace)",
                w.total, static_cast<size_t>(LAMP_NOALLOC_MAX_BYTES));
  void* ws = nullptr;
  if ((r = noalloc_base(&ws))) return r;
  // Every byte of the scratch that the attention reads is written first by the quantiser of
  // the same call, so nothing needs clearing between calls.
  return quant_and_attend(q, k, v, o, lse, ws, w, B, H, Hkv, Lq, Lk, D, causal, window, scale,
                          mask_bits, group_tiles, mode, tau, static_cast<cudaStream_t>(stream));
}

int lamp_check(void* stream) {
  LAMP_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize");
  uint32_t v = 0;
  LAMP_CUDA(cudaMemcpyFromSymbol(&v, lamp::g_lamp_error, sizeof(v)), "read error word");
  if (v) {
    const uint32_t zero = 0;
    LAMP_CUDA(cudaMemcpyToSymbol(lamp::g_lamp_error, &zero, sizeof(zero)), "clear error word");
    // A launch that gave up may leave its work-item counter held: wait for the device, then
    // return every scheduler slot of this device to idle.
    LAMP_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    {
      std::lock_guard<std::mutex> lk(g_sched_mu);
      unsigned long long* base = nullptr;
      if (int r = sched_base(&base)) return r;
      LAMP_CUDA(cudaMemset(base, 0, sizeof(lamp::g_lamp_sched)), "reset scheduler slots");
    }
    return fail(LAMP_ERR_TIMEOUT, "a device wait gave up (error word 0x%x, site %u)", v, (v >> 8) & 0xFFu);
  }
  return LAMP_OK;
}

int lamp_selftest_timeout(uint64_t wait_ns, void* stream) {
  if (wait_ns == 0 || wait_ns > 10000000000ull)
    return fail(LAMP_ERR_INVALID, "wait_ns must be in (0, 1e10]");
  lamp::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_ns);
  LAMP_CUDA(cudaGetLastError(), "selftest launch");
  return LAMP_OK;
}

int lamp_mma_probe(int kind, int n, int iters, void* stream) {
  if (kind < lamp::PROBE_F16_SS || kind > lamp::PROBE_F16_TS)
    return fail(LAMP_ERR_INVALID, "probe kind must be 0, 1 or 2");
  if (n != 64 && n != 128 && n != 256) return fail(LAMP_ERR_INVALID, "probe N must be 64, 128 or 256");
  if (iters < 1 || iters > (1 << 20)) return fail(LAMP_ERR_INVALID, "probe iters out of range");
  int nsm = 0;
  if (int r = sm_count(&nsm)) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kind == lamp::PROBE_F16_SS) return probe_n<lamp::PROBE_F16_SS>(n, nsm, iters, st);
  if (kind == lamp::PROBE_I8_SS) return probe_n<lamp::PROBE_I8_SS>(n, nsm, iters, st);
  return probe_n<lamp::PROBE_F16_TS>(n, nsm, iters, st);
}

const char* lamp_last_error(void) { return g_err; }

}  // extern "C"
