// kernels.h — internal launch interface between the C ABI layer (api.cu) and the
// kernel translation units.  Host code only; all pointers are device pointers and
// have been validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace nvfp4 {

// Launch with programmatic stream serialization (the kernel calls pdl_trigger and
// pdl_wait itself): the launch and the first CTAs of this kernel overlap the tail
// of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// CTAs of `kThreads` threads of kernel K that are resident at once on the current
// device (occupancy x SMs), looked up once per device: grid-stride kernels launch
// exactly one full wave.
template <auto K>
int resident_ctas(int threads) {
  // per device; host threads may race on the first call, all writing the same value
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    int per_sm = 0, sms = 148;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, K, threads, 0) != cudaSuccess) per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    n = (per_sm > 0 ? per_sm : 1) * sms;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// One wave of K, or fewer CTAs when `work` items (one per thread) need fewer.
template <auto K>
int wave_grid(int threads, int64_t work) {
  const int64_t want = (work + threads - 1) / threads;
  const int64_t cap = resident_ctas<K>(threads);
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

struct QuantizeArgs {
  const void* x;
  bool x_bf16;
  int64_t rows, cols, ldx;
  const float* gscale_in;  // nullable: one-pass mode with a supplied tensor scale
  uint8_t* codes;
  int64_t ld_codes;
  uint8_t* scales;
  int64_t ld_scales;
  bool sf_mma;
  float* gscale_out;
  float* amax_out;  // receives max|x| (required when gscale_in == nullptr)
  unsigned* status;
};
cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s);
// The amax pass of quantize alone (uses x, x_bf16, rows, cols, ldx, amax_out).
cudaError_t launch_amax(const QuantizeArgs& a, cudaStream_t s);

struct DequantizeArgs {
  const uint8_t* codes;
  int64_t ld_codes;
  const uint8_t* scales;
  int64_t ld_scales;
  bool sf_mma;
  const float* gscale;
  int64_t rows, cols;
  void* y;
  bool y_bf16;
  int64_t ldy;
};
cudaError_t launch_dequantize(const DequantizeArgs& a, cudaStream_t s);

struct KVLayout {
  uint8_t* base;
  int32_t heads, head_dim;
  int64_t chunk_tokens;
  int32_t max_chunks;
  int64_t off_k_codes, off_v_codes, off_k_scales, off_v_scales, off_mu, off_gscale, off_tokens, off_scratch;
  int64_t slot_codes_bytes, slot_scales_bytes;
};
int64_t kv_scratch_bytes(int32_t heads, int32_t head_dim, int64_t chunk_tokens);
// tokens: 1 .. chunk_tokens (a partial chunk fills the first tokens of the slot)
cudaError_t launch_kv_append(const KVLayout& c, const void* k, const void* v, int64_t tokens, int32_t slot,
                             unsigned* status, cudaStream_t s);
// Same append, but the statistics scratch is a static device array of the library
// (at most kNoAllocMaxColumns columns) instead of the cache's scratch region.
constexpr int64_t kNoAllocMaxColumns = 4096;
cudaError_t launch_kv_append_noalloc(const KVLayout& c, const void* k, const void* v, int64_t tokens,
                                     int32_t slot, unsigned* status, cudaStream_t s);
// tokens[i]: tokens held by slots[i] (checked on the device against the slot's
// recorded count); the output packs the slots' tokens in list order.
constexpr int kMaxWindowSlots = 64;
cudaError_t launch_kv_window(const KVLayout& c, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                             void* k_out, void* v_out, unsigned* status, cudaStream_t s);

// Attention scores of q [tq][heads][128] (bf16, row pitch ldq elements) against the
// window's keys, K dequantized from the cache inside the kernel; s_out [heads][tq][ld_s].
cudaError_t launch_kv_scores(const KVLayout& c, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                             const void* q, int64_t tq, int64_t ldq, float scale, void* s_out, bool s_bf16,
                             int64_t ld_s, unsigned* status, cudaStream_t s);

// Attention output O [tq][heads][128] (row pitch ldo) = P V^ over the window's keys,
// P bf16 [heads][tq][ld_p], V dequantized from the cache inside the kernel.
cudaError_t launch_kv_context(const KVLayout& c, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                              const void* p, int64_t tq, int64_t ld_p, void* o_out, bool o_bf16, int64_t ldo,
                              unsigned* status, cudaStream_t s);

// Test hook of the grid barrier of the one-launch quantization (see
// nvfp4_debug_grid_barrier): arrivals a barrier waits for beyond the grid's CTAs
// (0 = none) and its time limit (0 = the default 2 s).
void grid_barrier_debug(unsigned extra, unsigned long long limit_ns);
unsigned grid_barrier_extra();
unsigned long long grid_barrier_limit_ns();

// Zero n_words 32-bit words of device memory (a PDL-launched kernel, not a memset).
cudaError_t launch_zero_words(void* p, int n_words, cudaStream_t s);

constexpr int kMaxHistory = 1024;
cudaError_t launch_amax_history(float* history, int len, const float* amax_new, float* g_out, unsigned* status,
                                cudaStream_t s);

struct LoraArgs {
  const void* w;   // bf16 or fp32 [rows][ldw]
  bool w_bf16;
  int64_t rows, cols, ldw;
  const float* b;  // [rows][rank]
  const float* a;  // [rank][cols]
  int64_t rank;
  float scale;
  float* out;      // [rows][ldo]
  int64_t ldo;
};
cudaError_t launch_lora_merge(const LoraArgs& a, cudaStream_t s);

struct GemmOperand {
  const uint8_t* codes;
  int64_t ld_codes;
  const uint8_t* scales;  // MMA layout
  const float* gscale;
};
struct GemmArgs {
  GemmOperand a, w;
  int64_t M, N, K;
  void* c;        // nullable when q_codes is set
  bool c_bf16;
  int64_t ldc;
  int act;        // 0 none, 1 gelu(tanh)
  uint8_t* q_codes;  // fused requant output (nullable)
  int64_t q_ld_codes;
  uint8_t* q_scales;  // MMA layout
  const float* q_gscale_in;
  float* q_gscale_out;
  float* q_amax_out;  // nullable
  float* h_out;       // nullable
  unsigned* status;
};
cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t s);
// Test hook of the GEMM's bounded waits (see nvfp4_debug_gemm_fault).
void gemm_debug_fault(int drop_first_stage, unsigned long long wait_limit_ns);

}  // namespace nvfp4
