/*
 * nvfp4.h — C ABI of libnvfp4: NVFP4 activation quantization, the W4A4
 * block-scaled GEMM and the NVFP4 KV cache, for one sm_100a GPU.
 *
 * Sources (web pages describing LongLive-2.0; cited by title and section):
 *   [TW]  techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存"
 *         §一 "给AI视频生成做一次'瘦身手术'"  — the NVFP4 format: 4-bit E2M1 values,
 *             one FP8 scale per 16 values, one FP32 scale for the whole tensor.
 *         §三 "让视频一段一段'流水线式'地生成" — generation proceeds chunk by chunk
 *             (8 frames per chunk), each chunk appended to the KV cache.
 *         §四 "推理时三把'加速钥匙'" — all matmuls run in 4-bit (W4A4); the KV cache
 *             is stored in NVFP4 after subtracting the mean of K; a parallel CUDA
 *             kernel dequantizes several cache chunks of one window at once.
 *   [ZD]  github.zuobiaodaohang.com, "长视频生成的两堵物理墙" (NVlabs/LongLive write-up),
 *         section "NVFP4：数据体积砍到 1/4，带宽压力降一个数量级" — weights, activations
 *         and KV cache all 4-bit; the quantized KV cache is updated in place.
 *   [RM]  news.ainew.jp copy of the LongLive 2.0 README, "Quick Start / NVFP4" —
 *         weights are materialized once in NVFP4; quantized buffers must never be
 *         dtype-cast (so they cross this ABI as raw bytes).
 *
 * Number format (the readings this library fixes where the pages are silent):
 *   E2M1 code: bit 3 = sign, bits 0..2 index the magnitudes {0,0.5,1,1.5,2,3,4,6}.
 *   E4M3 block scale: OCP E4M3FN (bias 7, max 448, no Inf), one byte per 16
 *     consecutive values of a row, never negative, never NaN.
 *   Tensor scale g = RN_f32(amax / 2688), 2688 = 6 * 448, amax = max |x|.
 *   Block scale s = E4M3_RNE_satfinite(RN_f32(amax_block / RN_f32(6 * g))).
 *   Element code = sign(x) | E2M1 round-to-nearest-even of the EXACT quotient
 *     |x| / D with D = RN_f32(s * g), saturating at 6.  D == 0 gives magnitude 0.
 *   Decoded value = RN_f32(RN_f32(e2m1 * s) * g).
 *   Packing: element 2i of a row in the low nibble of byte i, 2i+1 in the high nibble.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory inside these calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and runs asynchronously.  Argument errors are detected on the host, return
 *     a status and enqueue nothing.
 *   - Data errors found on the device (a NaN/Inf input, a wait that gave up)
 *     set a sticky per-device status word (read it with nvfp4_get_device_status);
 *     the affected kernel then writes no output.  No kernel ever traps.
 *   - A device that is not compute capability 10.0 returns
 *     NVFP4_ERR_UNSUPPORTED_DEVICE.  There is no fallback path.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so this header needs no CUDA headers. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,        /* NULL pointer, bad enum, bad slot, overlap   */
  NVFP4_ERR_SHAPE = 2,              /* dimension mismatch or unsupported size      */
  NVFP4_ERR_ALIGNMENT = 3,          /* pointer or leading dimension misaligned     */
  NVFP4_ERR_NONFINITE = 4,          /* device status: a NaN or Inf input value     */
  NVFP4_ERR_TIMEOUT = 5,            /* device status: a bounded wait gave up       */
  NVFP4_ERR_CUDA = 6,               /* a CUDA runtime call failed                  */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 7  /* current device is not sm_100                */
} nvfp4_status;

typedef enum { NVFP4_BF16 = 0, NVFP4_FP32 = 1 } nvfp4_dtype;

/* Layout of the E4M3 block scales of an nvfp4_tensor.
 *   NVFP4_SF_ROWMAJOR: byte (r, j) at scales[r * ld_scales + j], j < cols/16.
 *   NVFP4_SF_MMA: the tensor-core operand layout.  Rows are grouped in tiles of
 *     128 and block-scale columns in groups of 4 (64 values of the row); each
 *     (row-tile, group) pair is one 512-byte atom, atoms stored row-tile-major:
 *       atom  = (r / 128) * ceil(cols / 64) + (j / 4)
 *       byte  = atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4)
 *     Total size nvfp4_scales_bytes(rows, cols, NVFP4_SF_MMA); padding bytes
 *     (rows beyond `rows`, groups beyond cols/16) are written as 0 by the
 *     library and must stay 0.  ld_scales is ignored.
 */
typedef enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_MMA = 1 } nvfp4_sf_layout;

/* One NVFP4 tensor [rows, cols] (cols % 16 == 0), all device memory:
 *   codes : rows * ld_codes bytes; ld_codes >= cols / 2, multiple of 16;
 *           base 16-byte aligned.
 *   scales: see nvfp4_sf_layout; base 16-byte aligned.
 *   gscale: one FP32 tensor scale g.
 * An empty tensor (rows == 0) may pass NULL codes and scales. */
typedef struct nvfp4_tensor {
  uint8_t* codes;
  uint8_t* scales;
  float* gscale;
  int64_t rows;
  int64_t cols;
  int64_t ld_codes;
  int64_t ld_scales;
  int32_t sf_layout; /* nvfp4_sf_layout */
  int32_t reserved;  /* must be 0 */
} nvfp4_tensor;

/* Bytes of the scale array of a [rows, cols] tensor in the given layout
 * (ROWMAJOR assumes ld_scales = cols / 16). */
nvfp4_status nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout, size_t* bytes);

/* nvfp4_quantize — activation (or weight) quantization to NVFP4.
 * [TW] §一 defines the format; [TW] §四 / [ZD] apply it to activations and weights.
 *   x        : device, row-major [rows, cols] of `xt` (NVFP4_BF16 or NVFP4_FP32),
 *              leading dimension ldx elements (ldx >= cols); base and row pitch
 *              16-byte aligned; may be NULL when rows == 0 (then g = 0, or the
 *              supplied g, and amax = 0).
 *   gscale_in: NULL  -> the tensor scale is computed from x: g = RN(amax / 2688)
 *                       (two passes over x). amax_out is then REQUIRED.
 *              !NULL -> device FP32 g used as given (one pass over x, e.g. a
 *                       scale calibrated on an earlier chunk).
 *   out      : rows/cols must match; codes, scales, gscale written; *out->gscale
 *              receives the g that was used.
 *   amax_out : device FP32, receives max|x| (nullable when gscale_in != NULL).
 * Errors: INVALID_ARG (NULL, bad dtype/layout), SHAPE (cols % 16, rows/cols
 * mismatch, ldx < cols), ALIGNMENT; device status NONFINITE if x holds NaN/Inf
 * (then nothing is written except amax_out). */
nvfp4_status nvfp4_quantize(const void* x, int32_t xt, int64_t rows, int64_t cols, int64_t ldx,
                            const float* gscale_in, const nvfp4_tensor* out, float* amax_out,
                            nvfp4_stream_t stream);

/* nvfp4_amax — max |x| over a whole tensor (the first step of quantization, alone).
 * [TW] §一: the tensor shares one FP32 scale; the library takes it as
 * g = RN(amax / 2688).  On its own this serves a tensor whose rows are split
 * across GPUs: each GPU takes the amax of its rows, the GPUs combine them with an
 * all-reduce(MAX) -- exact and independent of order; done on the binary32 bit
 * patterns as signed 32-bit integers it also carries a NaN through -- and each
 * quantizes its rows with nvfp4_quantize(gscale_in = RN(amax / 2688)), for which
 * nvfp4_amax_history_push with a one-entry history computes g on the device.  The
 * codes and scales of every row are then bit-identical to quantizing the whole
 * tensor on one GPU.
 *   x        : device, row-major [rows, cols] of xt (NVFP4_BF16 or NVFP4_FP32), ldx
 *              elements (>= cols), cols % 16 == 0; base and row pitch 16-byte
 *              aligned; may be NULL when rows == 0 (amax = 0).
 *   amax_out : device FP32 [1]: max|x| (its bits are those of the largest |x|, so
 *              an Inf gives +inf and a NaN a NaN).
 * Errors: INVALID_ARG (NULL, bad dtype), SHAPE, ALIGNMENT. */
nvfp4_status nvfp4_amax(const void* x, int32_t xt, int64_t rows, int64_t cols, int64_t ldx, float* amax_out,
                        nvfp4_stream_t stream);

/* nvfp4_dequantize — y = RN(RN(e2m1 * s) * g), stored as FP32 or as bf16 (RNE).
 * [TW] §一 (format).  y: device row-major [rows, cols], leading dimension ldy
 * elements, 16-byte aligned base and row pitch.  Either scale layout. */
nvfp4_status nvfp4_dequantize(const nvfp4_tensor* in, void* y, int32_t yt, int64_t ldy,
                              nvfp4_stream_t stream);

typedef enum { NVFP4_ACT_NONE = 0, NVFP4_ACT_GELU_TANH = 1 } nvfp4_activation;

/* Optional GEMM epilogue.
 *   act         : NVFP4_ACT_NONE or NVFP4_ACT_GELU_TANH,
 *                 h = 0.5 c (1 + tanh(sqrt(2/pi) (c + 0.044715 c^3))) in FP32.
 *   q_out       : non-NULL -> h is quantized to NVFP4 inside the GEMM (blocks of 16
 *                 along N) into q_out ([M, N], NVFP4_SF_MMA so that it can feed the
 *                 next GEMM as its A operand).  [AM] "scaling and quantization fused
 *                 into one kernel"; the tensor scale cannot be known before the
 *                 GEMM ends, so it is SUPPLIED:
 *   q_gscale_in : device FP32 g used for q_out (required with q_out; copied to
 *                 *q_out->gscale).
 *                 Non-finite h: a 16-block holding a NaN gets the E4M3 NaN scale
 *                 (0x7F) and codes that keep only the signs; a block with +-inf and
 *                 no NaN saturates (scale 448, code +-6 for the infinities).
 *   q_amax_out  : device FP32, nullable: receives max|h| (calibrates the next call);
 *                 NaN when h holds a NaN, so an amax history push rejects it.
 *   h_out       : device FP32 [M, N] (ld = N), nullable: also store h (verification).
 */
typedef struct nvfp4_epilogue {
  int32_t act;
  int32_t reserved;
  const nvfp4_tensor* q_out;
  const float* q_gscale_in;
  float* q_amax_out;
  float* h_out;
} nvfp4_epilogue;

/* nvfp4_gemm — C[m, n] = act(RN(acc[m, n] * RN(gA * gW))) with
 * acc = sum_k (e2m1(A) sA)(e2m1(W) sW) accumulated in FP32 by the tensor cores.
 * [TW] §四: the linear layers are the dominant cost and all run in 4-bit.
 *   A : [M, K] NVFP4, W : [N, K] NVFP4 (both K-major, i.e. row-major, both with
 *       sf_layout NVFP4_SF_MMA).  K % 64 == 0 is not required (the scale padding
 *       of the MMA layout is zero), K % 32 == 0 is (row pitch of codes).
 *   C : device row-major [M, N] of ct (FP32 or bf16), leading dimension ldc
 *       elements; may be NULL when the epilogue writes another output (q_out,
 *       h_out or q_amax_out).
 *   ep: nullable epilogue (activation, fused requantization).
 * Requires N % 16 == 0.  Errors: INVALID_ARG, SHAPE, ALIGNMENT; device status
 * TIMEOUT if a pipeline wait gave up. */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* W, void* C, int32_t ct,
                        int64_t ldc, const nvfp4_epilogue* ep, nvfp4_stream_t stream);

/* ---------------------------------------------------------------- KV cache ----
 * [TW] §四: K has its mean subtracted, then K and V are stored in NVFP4 (about
 * 1.125 bytes per K+V element pair vs 4 in bf16).  [TW] §三: chunks of tokens are
 * appended one by one; [ZD]: the cache is updated in place.
 * Reading fixed here: the mean mu is per (head, dim) over the chunk's tokens,
 *   mu = RN_f32(exact_sum / tokens), kept in FP32 and added back on dequant;
 *   K' = RN_f32(k - mu); one tensor scale per chunk for K' and one for V;
 *   16-value blocks run along head_dim.
 * Device layout of one cache (all inside the caller's allocation):
 *   k_codes [max_chunks][chunk_tokens][heads][head_dim/2]   (same for v_codes)
 *   k_scales[max_chunks][chunk_tokens][heads][head_dim/16]  (same for v_scales)
 *   mu      [max_chunks][heads][head_dim] FP32
 *   gscale  [max_chunks][2] FP32 (g_K, g_V)
 *   tokens  [max_chunks] int32: tokens held by each slot (written by every append)
 *   scratch used by kv_quant_append (per-column statistics of one chunk).
 * A slot may hold fewer tokens than chunk_tokens (a partial chunk, e.g. the last
 * chunk of a sequence or a sink chunk); its tokens are the first ones of the slot.
 */
typedef struct nvfp4_kv_cache {
  uint8_t* base;          /* device allocation given to nvfp4_kv_cache_init */
  size_t bytes;
  int32_t heads;
  int32_t head_dim;       /* multiple of 16 */
  int64_t chunk_tokens;
  int32_t max_chunks;
  int32_t reserved;
  int64_t off_k_codes, off_v_codes, off_k_scales, off_v_scales;
  int64_t off_mu, off_gscale, off_tokens, off_scratch;
  int64_t slot_codes_bytes;   /* chunk_tokens * heads * head_dim / 2  */
  int64_t slot_scales_bytes;  /* chunk_tokens * heads * head_dim / 16 */
} nvfp4_kv_cache;

/* Device bytes needed by a cache of the given geometry. */
nvfp4_status nvfp4_kv_cache_bytes(int32_t heads, int32_t head_dim, int64_t chunk_tokens,
                                  int32_t max_chunks, size_t* bytes);

/* Lays out a cache in caller-owned device memory `dev_mem` (256-byte aligned,
 * `bytes` >= nvfp4_kv_cache_bytes(...)) and fills the host struct `cache`.
 * No device work is enqueued; slots hold garbage until appended.
 * A caller that appends only with kv_quant_append_noalloc may give a shorter
 * allocation that ends at cache->off_scratch (the append scratch is then absent:
 * kv_quant_append returns NVFP4_ERR_INVALID_ARG on such a cache, while
 * kv_quant_append_noalloc and the window calls accept it).  Below off_scratch:
 * NVFP4_ERR_SHAPE. */
nvfp4_status nvfp4_kv_cache_init(void* dev_mem, size_t bytes, int32_t heads, int32_t head_dim,
                                 int64_t chunk_tokens, int32_t max_chunks, nvfp4_kv_cache* cache);

/* kv_quant_append — quantize one chunk of K and V into slot `slot`, in place.
 *   k, v   : device bf16 [tokens][heads][head_dim], 16-byte aligned.
 *   tokens : 1 .. cache->chunk_tokens; the mean mu is over these tokens and the
 *            slot records the count (a partial chunk holds its tokens first).
 * Appends to one cache must be issued on one stream (they share the scratch).
 * Device status NONFINITE on NaN/Inf input (the slot is then left unchanged). */
nvfp4_status kv_quant_append(const nvfp4_kv_cache* cache, const void* k, const void* v,
                             int64_t tokens, int32_t slot, nvfp4_stream_t stream);

/* kv_quant_append_noalloc — kv_quant_append for callers that cannot allocate
 * device memory.  No counterpart on the pages: it is a library convenience.
 * Some callers may not call cudaMalloc: a host framework that owns all device
 * memory through its own pool (a library allocation behind its back breaks its
 * accounting and fragments the pool), a real-time loop that must not stall on
 * the device-wide synchronization that cudaMalloc and cudaFree can imply, or a
 * plugin interface that hands a kernel only its input and output buffers.  This
 * entry point allocates nothing and needs no scratch from the caller: the
 * per-chunk column statistics live in one static device array of the library
 * (about 5 MiB, present on every device that loads the library until the
 * process exits), not in the cache's scratch region, which it never touches —
 * the cache may be laid out in an allocation that stops at off_scratch (see
 * nvfp4_kv_cache_init).
 * Inputs and outputs are exactly those of kv_quant_append and the slot it writes
 * is bit-identical.
 *   Limit: heads * head_dim <= NVFP4_NOALLOC_MAX_COLUMNS, else NVFP4_ERR_SHAPE.
 *   Set-up: the first call on a device looks up the array's device address for
 *   that device (the device current at the call); make that first call before
 *   any stream capture.
 *   Sharing: every call on a device uses the same array and it keeps the last
 *   call's contents; the call clears what must start at zero itself.  Calls whose
 *   work overlaps on the GPU (other streams, other threads) race on the array:
 *   issue them on one stream or serialize them.
 *   Device reset: the library keeps the array's device address (and that of the
 *   device status word) per device for the life of the process; after
 *   cudaDeviceReset on a device those cached addresses are stale, so do not call
 *   into the library on that device again in the same process. */
#define NVFP4_NOALLOC_MAX_COLUMNS 4096
nvfp4_status kv_quant_append_noalloc(const nvfp4_kv_cache* cache, const void* k, const void* v,
                                     int64_t tokens, int32_t slot, nvfp4_stream_t stream);

/* kv_dequant_window — dequantize the chunks listed in `slots_host` (a HOST array
 * of n_slots slot ids, 1 <= n_slots <= 64, repeats allowed, any order) in one
 * launch, writing bf16 [n_slots * chunk_tokens][heads][head_dim] to k_out and
 * v_out (device, 16-byte aligned) in list order:
 *   K^ = bf16(RN(RN(RN(e2m1 * s) * g_K) + mu)),  V^ = bf16(RN(RN(e2m1 * s) * g_V)).
 * Every listed slot must hold chunk_tokens tokens: a slot recorded with another
 * count sets device status NVFP4_ERR_SHAPE and its part of the output is not
 * written. */
nvfp4_status kv_dequant_window(const nvfp4_kv_cache* cache, const int32_t* slots_host,
                               int32_t n_slots, void* k_out, void* v_out,
                               nvfp4_stream_t stream);

/* kv_dequant_window_tokens — the same window over slots holding any number of
 * tokens, e.g. a sink-aware window: a sink slot, some shot-sink slots and the
 * sliding slots, possibly partial.  [TW] §四: one parallel kernel dequantizes the
 * window's chunks together; [TW] §六: global and shot-level anchor frames stay in
 * the attention range on top of the sliding window (a shot anchor is just a start
 * and a length, nothing is copied).
 *   tokens_host : HOST array, tokens_host[i] = tokens held by slots_host[i]
 *                 (1 .. chunk_tokens).
 * Output: bf16 [sum(tokens_host)][heads][head_dim], the slots' tokens one after
 * the other in list order.  A slot whose recorded count differs from the stated
 * one sets device status NVFP4_ERR_SHAPE and its part of the output is not
 * written. */
nvfp4_status kv_dequant_window_tokens(const nvfp4_kv_cache* cache, const int32_t* slots_host,
                                      const int32_t* tokens_host, int32_t n_slots, void* k_out,
                                      void* v_out, nvfp4_stream_t stream);

/* kv_window_scores — attention scores of a block of queries against the keys of a
 * window, reading K straight from the NVFP4 cache.  [TW] §四: the cache chunks of
 * the attention window are dequantized together and feed attention; here the
 * dequantization happens inside the kernel that computes Q K^T, one 128-key tile at
 * a time in shared memory, so no bf16 copy of the window's K is written to HBM.
 *   slots_host, tokens_host, n_slots : the window exactly as for
 *              kv_dequant_window_tokens (HOST arrays); Tk = sum(tokens_host) keys,
 *              in list order.
 *   q        : device bf16 [tq][heads][head_dim], row pitch ldq elements
 *              (ldq >= heads * head_dim); base and row pitch 16-byte aligned.
 *   scale    : FP32 factor applied to every score (e.g. 1 / sqrt(head_dim)).
 *   s_out    : device [heads][tq][ld_s] of st (NVFP4_FP32 or NVFP4_BF16), ld_s >= Tk,
 *              base and row pitch 16-byte aligned:
 *                S[h, i, j] = RN(scale * sum_d q[i, h, d] * K^[j, h, d]),
 *              the sum accumulated in FP32 by the tensor cores (bf16 products are
 *              exact), K^ bit for bit the window's K that kv_dequant_window_tokens
 *              writes; bf16 output is the RNE of that value.  Each row is written
 *              in whole 16-byte units: its elements from Tk up to the next 16-byte
 *              boundary receive 0 (inside the row, since ld_s * size is a multiple
 *              of 16); elements beyond that boundary are not written.
 * Requires head_dim == 128 (else NVFP4_ERR_SHAPE).  A listed slot whose recorded
 * token count differs sets device status NVFP4_ERR_SHAPE; its scores are then
 * unspecified.  Errors: INVALID_ARG (NULL, bad dtype or slot, non-finite scale),
 * SHAPE, ALIGNMENT. */
nvfp4_status kv_window_scores(const nvfp4_kv_cache* cache, const int32_t* slots_host, const int32_t* tokens_host,
                              int32_t n_slots, const void* q, int64_t tq, int64_t ldq, float scale, void* s_out,
                              int32_t st, int64_t ld_s, nvfp4_stream_t stream);

/* kv_window_context — the V side of attention from the NVFP4 cache: the weighted
 * sum of the window's values, O = P V^, with V dequantized inside the kernel (one
 * 64-key tile at a time, into shared memory; no bf16 copy of the window's V is
 * written).  [TW] §四, as for kv_window_scores.  When few query tiles face many
 * keys, the keys are split over the CTAs of a thread-block cluster (up to 8) and
 * their FP32 partial sums are added in a fixed order, so the result does not depend
 * on scheduling.
 *   slots_host, tokens_host, n_slots : the window (HOST arrays), Tk keys in list
 *              order, exactly as for kv_dequant_window_tokens.
 *   p        : device bf16 [heads][tq][ld_p] weights of the keys (e.g. the softmax
 *              of kv_window_scores' output), ld_p >= Tk; base and row pitch 16-byte
 *              aligned.  Elements beyond Tk in a row are not read.
 *   o_out    : device [tq][heads][head_dim] of ot (NVFP4_FP32 or NVFP4_BF16), row
 *              pitch ldo elements (>= heads * head_dim), base and pitch 16-byte aligned:
 *                O[i, h, d] = sum_j p[h, i, j] * V^[j, h, d],
 *              accumulated in FP32 by the tensor cores (and FP32 adds of partial
 *              sums), V^ bit for bit the window's V that kv_dequant_window_tokens
 *              writes; bf16 output is the RNE of it.
 * Requires head_dim == 128 and tq <= 65535 * 512.  A listed slot whose recorded token
 * count differs sets device status NVFP4_ERR_SHAPE (its keys then count as zero).
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT. */
nvfp4_status kv_window_context(const nvfp4_kv_cache* cache, const int32_t* slots_host, const int32_t* tokens_host,
                               int32_t n_slots, const void* p, int64_t tq, int64_t ld_p, void* o_out, int32_t ot,
                               int64_t ldo, nvfp4_stream_t stream);

/* ----------------------------------------------------------- amax history ----
 * A requantizing GEMM epilogue (nvfp4_epilogue.q_out) quantizes before its own
 * max|h| is known, so it takes a supplied tensor scale (q_gscale_in) and reports
 * max|h| (q_amax_out).  Reading fixed here for the steady state of chunk-by-chunk
 * generation ([TW] §三: chunks are generated one after another with the same
 * layers): keep the last `len` values of max|h| of a layer, newest first, and
 * supply g = RN(max(history) / 2688), the tensor-scale formula of quantize.
 * nvfp4_amax_history_push:
 *   history    : device fp32 [len], 1 <= len <= 1024 (zeros before the first push).
 *   amax_new   : device fp32, e.g. the previous call's q_amax_out.
 *   gscale_out : device fp32, the scale for the next call's q_gscale_in.
 * Shifts history by one, stores *amax_new in history[0], writes *gscale_out.  A
 * non-finite *amax_new sets device status NONFINITE and changes nothing. */
nvfp4_status nvfp4_amax_history_push(float* history, int32_t len, const float* amax_new, float* gscale_out,
                                     nvfp4_stream_t stream);

/* ------------------------------------------------------------- LoRA merge ----
 * github.zuobiaodaohang.com, "长视频生成的两堵物理墙", section "NVFP4：数据体积砍到 1/4":
 * "LoRA before quantization" — the LoRA is loaded into the weight first, then the
 * weight is quantized.  Reading fixed here (the page gives no formula): the usual
 * LoRA update in binary32 with one fixed order,
 *   acc = 0;  for j = 0 .. rank-1:  acc = RN(acc + RN(B[r][j] * A[j][c]));
 *   out[r][c] = RN(W[r][c] + RN(scale * acc)),
 * and the caller quantizes `out` with nvfp4_quantize (NVFP4_FP32 input).
 * nvfp4_lora_merge:
 *   w     : device [rows][ldw] of type wt (bf16 or fp32), ldw >= cols.
 *   lora_b: device fp32 [rows][rank] (row pitch rank);  lora_a: device fp32
 *           [rank][cols] (row pitch cols);  1 <= rank <= 4096.
 *   out   : device fp32 [rows][ldo], ldo >= cols; may not overlap w, lora_a or lora_b.
 * Errors: NULL pointers or rank outside 1..4096 -> INVALID_ARG; negative sizes or
 * pitches below cols -> SHAPE.  Non-finite values propagate into out (quantizing
 * it reports them).  rows == 0 or cols == 0 does nothing. */
nvfp4_status nvfp4_lora_merge(const void* w, nvfp4_dtype wt, int64_t rows, int64_t cols, int64_t ldw,
                              const float* lora_b, const float* lora_a, int32_t rank, float scale,
                              float* out, int64_t ldo, nvfp4_stream_t stream);

/* ----------------------------------------------------------------- status ----
 * Reads the sticky device status word of CUDA device `device` (synchronizes that
 * device first).  *status_out is NVFP4_OK or the first data error recorded since
 * the last clear; clear != 0 resets it to NVFP4_OK. */
nvfp4_status nvfp4_get_device_status(int32_t device, int32_t* status_out, int32_t clear);

/* Test hook for the bounded waits of the GEMM kernels (process-wide; no effect
 * until called).  Every wait of a GEMM kernel on a barrier gives up after a time
 * limit (2 s), records NVFP4_ERR_TIMEOUT in the device status word and lets the
 * kernel drain its own work and exit, so the context stays usable.
 *   drop_first_stage != 0: the TMA producer of every CTA skips its first pipeline
 *     stage, so the waits for that stage run out: the call ends with device
 *     status NVFP4_ERR_TIMEOUT and unspecified outputs.  0 restores normal work.
 *   wait_limit_ns > 0 replaces the 2 s limit of each wait; 0 restores it.
 * Not for use while other GEMM work is in flight. */
nvfp4_status nvfp4_debug_gemm_fault(int32_t drop_first_stage, uint64_t wait_limit_ns);

/* Test hook for the grid barrier of the one-launch quantization (a tensor that
 * fits in L2, tensor scale computed from the data), whose CTAs meet inside the
 * kernel between the amax pass and the encode pass (process-wide; no effect until
 * called).  Each barrier gives up after a time limit (2 s), records
 * NVFP4_ERR_TIMEOUT in the device status word and the kernel returns, so the
 * context stays usable.
 *   extra_arrivals > 0: every barrier waits for that many CTAs more than the grid
 *     has, so it runs out: the call ends with device status NVFP4_ERR_TIMEOUT and
 *     unspecified outputs.  0 restores normal work.
 *   wait_limit_ns > 0 replaces the 2 s limit; 0 restores it.
 * Not for use while other work of the library is in flight. */
nvfp4_status nvfp4_debug_grid_barrier(uint32_t extra_arrivals, uint64_t wait_limit_ns);

/* Human-readable name of a status code (static string). */
const char* nvfp4_status_string(int32_t status);

/* Library version, (major << 16) | minor. */
int32_t nvfp4_version(void);

/* Text of the CUDA error behind the last NVFP4_ERR_CUDA returned on the calling
 * thread ("no error" if none); a static string owned by the CUDA runtime. */
const char* nvfp4_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H_ */
