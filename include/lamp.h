/*
 * lamp.h -- C ABI of the tile-routed mixed-precision prefill attention library (B200, sm_100a).
 *
 * The operation (TileMix page, section 2 "How It Works"; LampAttention abstract):
 *   softmax attention O = softmax(scale * Q K^T) V, computed tile by tile over the score
 *   matrix.  Each (query tile, key tile) score tile is computed either from 8-bit per-block
 *   quantised Q and K (INT8 with fp32 block scales, or FP8 E4M3), then rescaled, or from the
 *   16-bit inputs.  The choice comes from a packed per-query-tile bitmask in which one bit
 *   governs a group of adjacent key tiles (0 = 16-bit, 1 = 8-bit; TileMix "Packed
 *   Bitmasks"), or from a look-ahead rule: a tile is recomputed in 16 bits when, for some row,
 *   its 8-bit tile max reaches the running row max minus tau (LampAttention).  Both paths
 *   update one online-softmax state per row; P.V is always 16-bit.
 *
 * Conventions for every call:
 *   - Pointers named q, k, v, o, lse, q8, k8, q_scale, k_scale, mask_bits, route_out are
 *     DEVICE pointers owned by the caller; the library keeps none of them after the call
 *     returns.  All device work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous.
 *   - Layouts are contiguous row-major: q, o [B][H][Lq][D]; k, v [B][Hkv][Lk][D]; lse
 *     [B][H][Lq]; q8 like q, k8 like k (one byte per element); q_scale [B][H][nQT];
 *     k_scale [B][Hkv][nKT]; mask_bits [B][H][nQT][W] uint64 words, bit g of a row at word
 *     g>>6, bit g&63 (LSB first).  nQT = ceil(Lq/BM), nKT = ceil(Lk/BN), W = ceil(nG/64),
 *     nG = ceil(nKT/group_tiles), with (BM, BN) from lamp_tile_shape(D).
 *   - q, k, v, q8, k8 must be 16-byte aligned (TMA) and o 32-byte aligned (32-byte stores);
 *     D must be 64, 128 or 256.
 *   - Return value: LAMP_OK or an error code.  Arguments are checked synchronously before
 *     anything is launched or any workspace is touched; on error nothing is enqueued and
 *     lamp_last_error() describes the problem (thread-local string).  Device-side failures (a bounded wait in a kernel that
 *     gave up) are reported by lamp_check().
 */
#ifndef LAMP_H
#define LAMP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  LAMP_OK = 0,
  LAMP_ERR_INVALID = 1,      /* bad argument (null pointer, size, alignment, H % Hkv)      */
  LAMP_ERR_UNSUPPORTED = 2,  /* valid but not implemented here (D, window without causal) */
  LAMP_ERR_CUDA = 3,         /* a CUDA runtime call failed                                */
  LAMP_ERR_TIMEOUT = 4       /* a device-side bounded wait gave up (see lamp_check)       */
};

/* mode bit field */
#define LAMP_ROUTE_BITMASK 0x0u  /* bit 0: routing from mask_bits (TileMix)               */
#define LAMP_ROUTE_ADAPTIVE 0x1u /* bit 0: look-ahead rule with threshold tau (Lamp)      */
#define LAMP_FMT_INT8 0x0u       /* bit 1: 8-bit format INT8, scale = absmax/127          */
#define LAMP_FMT_E4M3 0x2u       /* bit 1: 8-bit format FP8 E4M3, scale = absmax/448      */
#define LAMP_IN_FP16 0x0u        /* bit 2: q, k, v are fp16                               */
#define LAMP_IN_BF16 0x4u        /* bit 2: q, k, v are bf16                               */
#define LAMP_OUT_F32 0x0u        /* bit 3: o is fp32                                      */
#define LAMP_OUT_INDTYPE 0x8u    /* bit 3: o has the input dtype                          */
#define LAMP_PV_E4M3 0x10u       /* bit 4: 8-bit exponentials and an 8-bit P.V (below)     */

/* Routing tile (BM x BN) for head dimension D: 64 -> 64x64, 128 -> 128x128, 256 -> 64x128
 * (TileMix "The Tile Architecture": hardware-aligned score tiles of 128x128 or 64x64).
 * Returns LAMP_OK, or LAMP_ERR_UNSUPPORTED for any other D.  bm/bn may not be NULL. */
int lamp_tile_shape(int D, int* bm, int* bn);

/* Number W of uint64 mask words per query tile (TileMix "Packed Bitmasks", grouping of
 * adjacent key tiles): W = ceil(ceil(nKT / group_tiles) / 64).  Returns W > 0, or -1 when the
 * arguments are invalid (Lk < 1, group_tiles < 1, unsupported D). */
int lamp_mask_words(int Lk, int D, int group_tiles);

/* Per-block quantisation of Q and K to 8 bits (TileMix "The Dual-Path Engine", item 2;
 * LampAttention "8-bit formats").  For every (batch, head) block of BM query rows (Q) or BN
 * key rows (K) over all D channels: a = max |x|; scale = fl32(a / 127) (INT8) or
 * fl32(a / 448) (E4M3); code = RNE(fl32(x / scale)), clamped to [-127, 127] (INT8) or
 * saturated to +-448 (E4M3); an all-zero block gets scale 0 and zero codes.
 * q8/k8 receive int8 two's complement or e4m3 bytes; q_scale/k_scale the fp32 scales.
 * mode: LAMP_FMT_* | LAMP_IN_*; other bits ignored.  k/k8/k_scale may all be NULL to
 * quantise Q only (and q/q8/q_scale NULL for K only). */
int lamp_quant_qk(const void* q, const void* k, void* q8, void* k8, float* q_scale,
                  float* k_scale, int B, int H, int Hkv, int Lq, int Lk, int D, int mode,
                  void* stream);

/* 8-bit V for the 8-bit P.V mode (LampAttention abstract: the exponentials are evaluated in
 * 8-bit formats; the pages fix no format, and this library reads it as E4M3 for both P and V).
 * One scale per (batch, KV head, channel) over all Lk keys: a = max_j |v_jd|, v_scale =
 * fl32(a / 448), code = E4M3(fl32(v / v_scale)) rounded to nearest even (a = 0: scale 0 and
 * zero codes).  v: [B][Hkv][Lk][D] 16-bit (mode: LAMP_IN_*); v8t: [B][Hkv][D][Lk16] E4M3
 * codes, channel-major, Lk16 = Lk rounded up to a multiple of 16 (the padding written as
 * zero), 16-byte aligned; v_scale: [B][Hkv][D] fp32.  D: 64, 128 or 256.  Three kernels (channel
 * maxima into v_scale, codes, maxima -> scales) on `stream`. */
int lamp_quant_v(const void* v, void* v8t, float* v_scale, int B, int Hkv, int Lk, int D,
                 int mode, void* stream);

/* Seeded routing template (TileMix: routing policies are static, data-free templates; the
 * template's shape is not given, so each group bit is an independent draw).  Bit g of the
 * mask of (b, h, qt) is 0 (16-bit) with probability fp16_fraction:
 *   u = splitmix64(seed XOR idx * 0x9E3779B97F4A7C15), idx = ((b*H + h)*nQT + qt)*nG + g,
 *   bit = ((u >> 11) * 2^-53 < fp16_fraction) ? 0 : 1; bits g >= nG are 0.
 * splitmix64(x) is one step of Steele-Lea-Flood SplitMix64 from state x.
 * mask_bits: device buffer of B*H*nQT*W uint64 words, fully written. */
int lamp_build_mask(uint64_t* mask_bits, int B, int H, int Lq, int Lk, int D, int group_tiles,
                    float fp16_fraction, uint64_t seed, void* stream);

/* Structured static routing template (TileMix page, section 4: the routing policy is a
 * static, data-free structured template; section 3: the "SpTrans75" configuration routes 75%
 * of the work to INT8).  The pages give no shape; this one follows the local and strided
 * layouts of sparse transformers.  For routing row qt (BM query rows) the diagonal key tile
 *   kd = clamp((min(Lq, (qt+1)*BM) - 1 + Lk - Lq) / BN, 0, nKT - 1),   gd = kd / group_tiles
 * holds the key aligned with the row's last query (bottom-right), and group g is 16-bit
 * (bit 0) iff g < sink_groups, or |gd - g| < band_groups, or stride_groups > 0 divides
 * |gd - g|; every other group is 8-bit (bit 1); bits g >= nG are 0.  Every (batch, head)
 * gets the same template.  mask_bits: device buffer of B*H*nQT*W uint64 words, fully
 * written.  Negative template parameters return LAMP_ERR_INVALID. */
int lamp_build_mask_template(uint64_t* mask_bits, int B, int H, int Lq, int Lk, int D,
                             int group_tiles, int sink_groups, int band_groups,
                             int stride_groups, void* stream);

/* Host-side, no GPU work: the fraction of visible (query, key) pairs of one (batch, head)
 * that the template above routes to 16 bits, with the causal / window limits of
 * lamp_attn_fwd_q8.  Writes *fp16_fraction (0 when no pair is visible); LAMP_ERR_INVALID for
 * invalid sizes, parameters or a NULL output. */
int lamp_template_fraction(int Lq, int Lk, int D, int group_tiles, int causal, int window,
                           int sink_groups, int band_groups, int stride_groups,
                           double* fp16_fraction);

/* Host-side, no GPU work: template parameters whose 8-bit share of the visible pairs is
 * closest to int8_fraction (0.75 for the pages' SpTrans75), searched over sink_groups in
 * {1, 0}, stride_groups in {0, 2, 3, ..., nG}, band_groups in {1, ..., nG} (the first best in
 * that order).  Writes the three parameters and the realised 16-bit fraction; NULL outputs
 * or int8_fraction outside [0, 1] return LAMP_ERR_INVALID. */
int lamp_template_for_int8_fraction(int Lq, int Lk, int D, int group_tiles, int causal,
                                    int window, double int8_fraction, int* sink_groups,
                                    int* band_groups, int* stride_groups,
                                    double* fp16_fraction);

/* Routed attention forward, end to end: quantises Q and K into the library workspace, then
 * runs the routed attention kernel.  Arguments as lamp_attn_fwd_q8 without the 8-bit operands.
 * o receives O (fp32, or the input dtype with LAMP_OUT_INDTYPE); lse receives the natural-log
 * row log-sum-exp of the scaled, routed scores (may be NULL).  Rows that see no key get
 * O = 0 and lse = -inf.
 * Workspace: the caller's (lamp_set_workspace), else one cached block per device that is
 * grown in stream order on `stream` (cudaMallocAsync, the old block released with
 * cudaFreeAsync behind the work already queued there), so growing it never synchronises the
 * device.  Calls that share the workspace must not overlap on the GPU: calls on different
 * streams need the caller's ordering (events) between them.
 * Every argument check of lamp_attn_fwd_q8 runs before the workspace is touched or anything
 * is enqueued. */
int lamp_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int Hkv, int Lq, int Lk, int D, int causal, int window, float scale,
                  const uint64_t* mask_bits, int group_tiles, int mode, float tau, void* stream);

/* Routed attention forward on already-quantised operands (the attention kernel alone).
 *   causal: 0/1, bottom-right aligned (query i sees key j iff j <= i + Lk - Lq);
 *   window: > 0 keeps only the `window` most recent keys (j > i + Lk - Lq - window); needs
 *           causal = 1, else LAMP_ERR_UNSUPPORTED;
 *   scale:  softmax scale applied to q.k; <= 0 means 1/sqrt(D);
 *   mask_bits/group_tiles: bitmask routing; mask_bits NULL = every tile 8-bit; ignored in
 *           adaptive mode;
 *   tau:    adaptive threshold in natural-log units of the scaled score; ignored in bitmask
 *           mode;
 *   route_out: optional device buffer uint8 [B][H][nQT][nKT] receiving the routing decision
 *           of every tile: 0 = no visible pair, 1 = 8-bit, 2 = 16-bit by mask, 3 = 16-bit by
 *           the look-ahead rule (4 = dropped, lamp_attn_fwd_q8_skip).  NULL to skip.
 * GQA: query head h reads KV head h / (H / Hkv). */
int lamp_attn_fwd_q8(const void* q, const void* k, const void* v, const void* q8,
                     const void* k8, const float* q_scale, const float* k_scale, void* o,
                     float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                     int window, float scale, const uint64_t* mask_bits, int group_tiles,
                     int mode, float tau, uint8_t* route_out, void* stream);

/* Debug capture of the routed attention kernel (parity checks and measurement; the pages have
 * no counterpart).  Runs the kernel and launch configuration that lamp_attn_fwd_q8 runs for the
 * same arguments (dense batches, no threshold skip), in an instantiation that also copies raw
 * score tiles out, and writes o, lse and route_out as lamp_attn_fwd_q8 does:
 *   tile_slot: device int32 [B][H][nQT][nKT]; a value s in [0, n_slots) selects routing tile
 *              (b, h, qt, kt) for slot s; any other value leaves the tile out;
 *   s8_dump:   device 32-bit words [n_slots][BM][BN], or NULL: the tile's 8-bit product as the
 *              kernel read it from tensor memory, before any scaling or masking -- the int32
 *              accumulators sum_d cq[i][d] * ck[j][d] (INT8) or their fp32 bits (E4M3) -- for
 *              every tile scored in 8 bits (route codes 1 and 3: the look-ahead rule's 8-bit
 *              pass of a recomputed tile included);
 *   s16_dump:  device fp32 [n_slots][BM][BN], or NULL: the unscaled 16-bit product
 *              sum_d q[i][d] * k[j][d] of every tile scored in 16 bits (route codes 2 and 3).
 * Rows i >= Lq and keys j >= Lk of a tile hold the product of the zero padding (0).  Slots of
 * tiles without such a product are left as they were.  The dump buffers must be 16-byte
 * aligned; LAMP_ERR_INVALID for a NULL slot map, n_slots < 1 or no dump buffer. */
int lamp_attn_debug(const void* q, const void* k, const void* v, const void* q8,
                    const void* k8, const float* q_scale, const float* k_scale, void* o,
                    float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                    int window, float scale, const uint64_t* mask_bits, int group_tiles,
                    int mode, float tau, uint8_t* route_out, const int* tile_slot, int n_slots,
                    void* s8_dump, void* s16_dump, void* stream);

/* The kernels' exponentials on n inputs (tests and measurement; the pages have no counterpart):
 * y[i] = 2^x[i] by method 0, the degree-3 polynomial on the FMA pipe that the single-tile
 * kernel uses for one exponential pair in eight (range reduction to [-1/2, 1/2] with the
 * round-to-nearest constant 1.5 * 2^23; relative error below 7.7e-5 for x in [-125, 0]; 0 below
 * -125), or method 1, the hardware approximation ex2.approx.ftz.  x, y: device fp32 arrays. */
int lamp_exp2_eval(const float* x, float* y, int n, int method, void* stream);

/* Same operation and arguments as lamp_attn_fwd, for callers that cannot allocate device
 * memory: code whose device memory is all owned by another allocator (a framework's caching
 * allocator that has already reserved it), or latency-bound serving loops that must not call
 * cudaMalloc / cudaFree, which may synchronise the whole device and take unbounded time.
 * This entry point allocates nothing.  (The pages have no counterpart to it.)
 *   - Scratch for the 8-bit Q, K and their block scales lives in one file-scope device array
 *     of LAMP_NOALLOC_MAX_BYTES, which every GPU that loads this library holds until the
 *     process exits.  Problems needing more (lamp_workspace_size(...) > the maximum) are
 *     rejected with LAMP_ERR_INVALID before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.  With CUDA's
 *     lazy module loading, the first lamp_* call that needs this library's device code on a
 *     device (a kernel launch, or that lookup) loads the module there, and loading it is when
 *     the driver places the array and the code in device memory.  Callers that must not see
 *     any allocation after their set-up make one such call (this one, on a small problem)
 *     during set-up.
 *   - All calls share the one array and it keeps the last call's contents; every byte a call
 *     reads is written earlier in the same call, so nothing needs clearing.  Calls whose work
 *     overlaps on the GPU (different streams, no ordering between them) race on the array.
 *   - The caller still passes (and owns) q, k, v, o, lse and mask_bits. */
#define LAMP_NOALLOC_MAX_BYTES (32u << 20)
int lamp_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int Hkv, int Lq, int Lk, int D, int causal, int window,
                          float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                          float tau, void* stream);

/* lamp_attn_fwd on HOST buffers, with the host-device copies pipelined against the compute
 * (no counterpart in the pages: a runtime entry point for callers whose Q, K, V live in host
 * memory and who want O back there).  q, k, v: host [B][H|Hkv][L][D] 16-bit; o: host
 * [B][H][Lq][D] (fp32, or the input dtype with LAMP_OUT_INDTYPE); lse: host [B][H][Lq] fp32 or
 * NULL; host buffers need no alignment, and only page-locked (pinned) ones let the copies
 * overlap the compute.  mask_bits stays a DEVICE buffer (as for lamp_attn_fwd).  Every other
 * argument, every check and every result bit is as lamp_attn_fwd's.
 * The B * Hkv KV planes (each KV head with its H / Hkv query heads: independent problems) are
 * cut into n_chunks chunks of consecutive planes (0: about 256 MB of copies per chunk, at most
 * 8; clamped to [1, B * Hkv]).  Per chunk: Q, K, V are copied in on a library copy stream,
 * quantised and attended on `stream`, and O, lse copied out on a second copy stream, through
 * two device buffer slots in the library workspace (two chunks' inputs and outputs plus one
 * chunk's 8-bit codes), so that chunk c + 1 is copied in and chunk c - 1 copied out while
 * chunk c computes.  The copy streams start behind the work queued on `stream` before the
 * call, and `stream` continues only once every copy of the call has completed; the host
 * buffers must stay valid until then.  Calls on different streams share the workspace and
 * the copy streams: they need the caller's ordering between them.  Argument errors return
 * before anything is enqueued. */
int lamp_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int Hkv, int Lq, int Lk, int D, int causal, int window,
                       float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                       float tau, int n_chunks, void* stream);

/* The routed attention kernel with 8-bit exponentials and an 8-bit P.V (mode must include
 * LAMP_PV_E4M3; D = 128; dense batches; no threshold skip).  As lamp_attn_fwd_q8, except that
 * V is given as lamp_quant_v's v8t / v_scale (no 16-bit V).  Per row, in ascending key tiles:
 * the running max m_t after tile t (of the routed scores, as in the 16-bit P mode), each
 * p = 2^(x - m_t) * 2^8 rounded to E4M3 (the row max's p is 256), P.V = the E4M3 MMA of P and
 * V's codes, and O = v_scale * sum p8 v8 / sum p8 (the tiles rescaled to the final max); lse
 * is that of the exact p.  Runs on the single-tile kernel. */
int lamp_attn_fwd_q8_pv8(const void* q, const void* k, const void* q8, const void* k8,
                         const float* q_scale, const float* k_scale, const void* v8t,
                         const float* v_scale, void* o, float* lse, int B, int H, int Hkv,
                         int Lq, int Lk, int D, int causal, int window, float scale,
                         const uint64_t* mask_bits, int group_tiles, int mode, float tau,
                         void* stream);

/* Look-ahead routing with a threshold skip (LampAttention abstract: 8-bit products decide which
 * sub-blocks need 16 bits; LATTE page: low-precision dot products filter out the keys far below
 * the row maximum).  As lamp_attn_fwd_q8 in look-ahead mode (mode must hold
 * LAMP_ROUTE_ADAPTIVE; no mask), plus: a live routing tile is dropped -- it contributes
 * nothing to m, l or O -- iff every row with a visible key in it has a running max m_r and
 * its 8-bit tile max t_r < m_r - skip_tau; kept tiles follow the look-ahead rule with tau.
 * skip_tau is in natural-log units, tau <= skip_tau; +inf disables the skip.  A query tile's
 * first live key tile is never dropped.  route_out marks dropped tiles 4.
 * LAMP_ERR_INVALID for a NaN skip_tau, skip_tau < tau or a mode without LAMP_ROUTE_ADAPTIVE. */
int lamp_attn_fwd_q8_skip(const void* q, const void* k, const void* v, const void* q8,
                          const void* k8, const float* q_scale, const float* k_scale, void* o,
                          float* lse, int B, int H, int Hkv, int Lq, int Lk, int D, int causal,
                          int window, float scale, int mode, float tau, float skip_tau,
                          uint8_t* route_out, void* stream);

/* Decode with an 8-bit key/value cache (TileMix page, section 4: INT8 key/value caches for the
 * decode phase; GQA).  One new query row per (batch, head) attends to the first len_k[b]
 * cached keys of its sequence (all max_k when len_k is NULL):
 *   q: [B][H][D] 16-bit; q8 / q_scale: its 8-bit codes and per-row scales, as lamp_quant_qk
 *      writes them with Lq = 1 ([B][H][D], [B][H]);
 *   k8, v8: [B][Hkv][max_k][D] 8-bit cache codes; k_scale, v_scale: [B][Hkv][ceil(max_k/BN)]
 *      per-block scales (lamp_quant_qk on K, and on V in K's place);
 *   mask_bits: [B][H][1][W], W = lamp_mask_words(max_k, D, group_tiles), or NULL (every group
 *      8-bit).  Bit 1: s = (q8 . k8) * sq * sk * scale.  Bit 0 (16-bit route): s =
 *      (q . k8) * sk * scale, the full-precision query against the dequantised cached key (the
 *      cache holds no 16-bit keys);
 *   values v8 * sv; softmax and P.V in fp32; o: [B][H][D] fp32; lse: [B][H] natural log, -inf
 *      for an empty cache.
 * mode: LAMP_FMT_*, LAMP_IN_* (bitmask routing, fp32 output; else LAMP_ERR_UNSUPPORTED); at
 * most 8 query heads per KV head.  Uses the library workspace (B * H * ceil(max_k / 1024) *
 * (D + 2) floats of split partials: one per run of 8 chunks of 128 keys), like lamp_attn_fwd. */
int lamp_decode_fwd(const void* q, const void* q8, const float* q_scale, const void* k8,
                    const float* k_scale, const void* v8, const float* v_scale, const int* len_k,
                    float* o, float* lse, int B, int H, int Hkv, int max_k, int D, float scale,
                    const uint64_t* mask_bits, int group_tiles, int mode, void* stream);

/* ---- variable-length batches (TileMix page, section 4: GQA and variable-length batches
 * are supported) --------------------------------------------------------------------------
 * B sequences of different lengths share one launch.  Sequence b owns query rows
 * [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]); cu_q / cu_k are device int32 arrays
 * of B + 1 non-decreasing offsets with cu_q[0] = cu_k[0] = 0, cu_q[B] = total_q, cu_k[B] =
 * total_k, and no sequence longer than max_q / max_k.  Sequences are independent problems:
 * causal and window limits, routing tiles and quantisation blocks all start at each
 * sequence's first row (bottom-right causal alignment within the sequence).
 * Layouts (head-major, rows packed):
 *   q, q8, o: [H][total_q][D];  k, v, k8: [Hkv][total_k][D];  lse: [H][total_q];
 *   q_scale:  [B][H][ceil(max_q/BM)];  k_scale: [B][Hkv][ceil(max_k/BN)] (entries past a
 *             sequence's own block count are 0);
 *   mask_bits: [B][H][ceil(max_q/BM)][W], W = lamp_mask_words(max_k, D, group_tiles), the
 *             layout lamp_build_mask(mask, B, H, max_q, max_k, ...) writes; route_out
 *             likewise [B][H][ceil(max_q/BM)][ceil(max_k/BN)].
 * Offsets are read on the device; a sequence whose offsets are decreasing or longer than
 * max_q / max_k is clipped to [0, max] rows and never written past total_q. */
int lamp_quant_qk_varlen(const void* q, const void* k, void* q8, void* k8, float* q_scale,
                         float* k_scale, const int* cu_q, const int* cu_k, int B, int H,
                         int Hkv, int max_q, int max_k, int total_q, int total_k, int D,
                         int mode, void* stream);
int lamp_attn_fwd_q8_varlen(const void* q, const void* k, const void* v, const void* q8,
                            const void* k8, const float* q_scale, const float* k_scale,
                            void* o, float* lse, const int* cu_q, const int* cu_k, int B, int H,
                            int Hkv, int max_q, int max_k, int total_q, int total_k, int D,
                            int causal, int window, float scale, const uint64_t* mask_bits,
                            int group_tiles, int mode, float tau, uint8_t* route_out,
                            void* stream);
/* Quantise (into the library workspace, as lamp_attn_fwd) and run the routed attention on
 * a variable-length batch. */
int lamp_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int* cu_q, const int* cu_k, int B, int H, int Hkv, int max_q,
                         int max_k, int total_q, int total_k, int D, int causal, int window,
                         float scale, const uint64_t* mask_bits, int group_tiles, int mode,
                         float tau, void* stream);

/* Bytes of workspace lamp_attn_fwd needs for these sizes (q8, k8 and the scales, each
 * 256-byte aligned).  0 on invalid arguments. */
size_t lamp_workspace_size(int B, int H, int Hkv, int Lq, int Lk, int D, int mode);

/* Give the library a caller-owned device workspace (ptr may be NULL to drop it and return
 * to the cached allocation).  The library uses it for every later lamp_attn_fwd on any
 * stream until replaced; the caller keeps ownership and must keep it alive. */
int lamp_set_workspace(void* ptr, size_t bytes);

/* Synchronises `stream`, then reports and clears the device-side error word: LAMP_OK, or
 * LAMP_ERR_TIMEOUT when a kernel's bounded wait gave up since the last check (the kernel
 * then stopped early and its outputs are undefined), or LAMP_ERR_CUDA.  After a timeout it
 * also synchronises the device and returns the attention kernel's work-item counters to
 * idle (a launch that gave up may have left one held), so call it while no other call of
 * the library is running on the device. */
int lamp_check(void* stream);

/* Launches a one-block kernel that waits, with a limit of `wait_ns` nanoseconds, on a
 * barrier nothing will ever complete, so that the bounded-wait error path can be tested
 * without faulting or hanging the GPU.  A later lamp_check() returns LAMP_ERR_TIMEOUT. */
int lamp_selftest_timeout(uint64_t wait_ns, void* stream);

/* Tensor-core throughput probe (measurement only; the pages have no counterpart): launches one
 * CTA per SM on `stream`; the CTA's elected thread issues iters x 8 back-to-back tcgen05 MMAs of
 * M = 128, N = n into one TMEM accumulator, with descriptors built once, and waits for them.
 * kind: 0 = kind::f16 bf16 with A and B in shared memory (K = 16 per MMA), 1 = kind::i8 with A
 * and B in shared memory (K = 32), 2 = kind::f16 bf16 with A in tensor memory and B in shared
 * memory (K = 16).  Operands are zero.  Work = 2 * 128 * n * K * 8 * iters operations per SM;
 * the caller times the launch (CUDA events on `stream`).  n: 64, 128 or 256; iters in
 * [1, 2^20].  Returns LAMP_OK or LAMP_ERR_INVALID / LAMP_ERR_CUDA. */
int lamp_mma_probe(int kind, int n, int iters, void* stream);

/* Thread-local description of the last error returned by a lamp_* call on this thread. */
const char* lamp_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LAMP_H */
