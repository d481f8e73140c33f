// kernels.h — internal launch interface between the C ABI layer (api.cu) and the
// kernel translation units.  Host code only; all pointers are device pointers and
// have been validated by the caller.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

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
  int64_t off_k_codes, off_v_codes, off_k_scales, off_v_scales, off_mu, off_gscale, off_scratch;
  int64_t slot_codes_bytes, slot_scales_bytes;
};
int64_t kv_scratch_bytes(int32_t heads, int32_t head_dim, int64_t chunk_tokens);
cudaError_t launch_kv_append(const KVLayout& c, const void* k, const void* v, int32_t slot,
                             unsigned* status, cudaStream_t s);
// Same append, but the statistics scratch is a static device array of the library
// (at most kNoAllocMaxColumns columns) instead of the cache's scratch region.
constexpr int64_t kNoAllocMaxColumns = 4096;
cudaError_t launch_kv_append_noalloc(const KVLayout& c, const void* k, const void* v, int32_t slot,
                                     unsigned* status, cudaStream_t s);
cudaError_t launch_kv_window(const KVLayout& c, const int32_t* slots, int32_t n_slots, void* k_out,
                             void* v_out, cudaStream_t s);

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

}  // namespace nvfp4
