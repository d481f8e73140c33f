// api.cu — the libnvfp4 C ABI: argument validation, device checks, the sticky
// device status word, and dispatch to the kernels.  Every entry point is declared
// and documented in include/nvfp4.h.
#include <mutex>

#include "kernels.h"
#include "nvfp4.h"

static_assert(NVFP4_NOALLOC_MAX_COLUMNS == nvfp4::kNoAllocMaxColumns,
              "header and library agree on the static scratch limit");

// One status word per device (a module global: every device that loads the
// library holds its own copy).  Kernels record the first data error here.
__device__ unsigned nvfp4_device_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices];
int g_dev_state[kMaxDevices];  // 0 unknown, 1 supported, -1 unsupported

nvfp4_status init_device(int dev, unsigned** status) {
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_dev_state[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) {
      g_dev_state[dev] = -1;
    } else {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, nvfp4_device_status_word) != cudaSuccess) return NVFP4_ERR_CUDA;
      g_status_ptr[dev] = static_cast<unsigned*>(p);
      g_dev_state[dev] = 1;
    }
  }
  if (g_dev_state[dev] < 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  *status = g_status_ptr[dev];
  return NVFP4_OK;
}

nvfp4_status current_device(unsigned** status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  return init_device(dev, status);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The CUDA error behind the last NVFP4_ERR_CUDA returned on this thread.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

nvfp4_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  g_last_cuda_error = e;
  return NVFP4_ERR_CUDA;
}

constexpr int64_t kMaxBlocks = (int64_t)1 << 31;

int64_t sf_mma_bytes(int64_t rows, int64_t cols) {
  return (rows + 127) / 128 * 128 * ((cols / 16 + 3) / 4) * 4;
}

// Checks common to every nvfp4_tensor argument.
nvfp4_status check_tensor(const nvfp4_tensor* t) {
  if (!t || !t->gscale) return NVFP4_ERR_INVALID_ARG;
  if (t->rows > 0 && (!t->codes || !t->scales)) return NVFP4_ERR_INVALID_ARG;  // empty: may be NULL
  if (t->reserved != 0) return NVFP4_ERR_INVALID_ARG;
  if (t->sf_layout != NVFP4_SF_ROWMAJOR && t->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
  if (t->rows < 0 || t->cols <= 0 || t->cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (t->ld_codes < t->cols / 2 || t->ld_codes % 16 != 0) return NVFP4_ERR_SHAPE;
  if (t->sf_layout == NVFP4_SF_ROWMAJOR && t->ld_scales < t->cols / 16) return NVFP4_ERR_SHAPE;
  if (!aligned16(t->codes) || !aligned16(t->scales) || (reinterpret_cast<uintptr_t>(t->gscale) & 3u))
    return NVFP4_ERR_ALIGNMENT;
  const int64_t vblocks = (t->rows + 127) / 128 * 128 * ((t->cols / 16 + 3) / 4 * 4);
  if (vblocks >= kMaxBlocks) return NVFP4_ERR_SHAPE;
  return NVFP4_OK;
}

bool valid_dtype(int32_t t) { return t == NVFP4_BF16 || t == NVFP4_FP32; }

}  // namespace

extern "C" {

int32_t nvfp4_version(void) { return (1 << 16) | 0; }

const char* nvfp4_last_cuda_error_string(void) {
  return g_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(g_last_cuda_error);
}

const char* nvfp4_status_string(int32_t s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "unsupported or mismatched shape";
    case NVFP4_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_NONFINITE: return "non-finite input value";
    case NVFP4_ERR_TIMEOUT: return "a device wait gave up";
    case NVFP4_ERR_CUDA: return "CUDA runtime error";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    default: return "unknown status";
  }
}

nvfp4_status nvfp4_scales_bytes(int64_t rows, int64_t cols, int32_t sf_layout, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (sf_layout == NVFP4_SF_ROWMAJOR) *bytes = (size_t)(rows * (cols / 16));
  else if (sf_layout == NVFP4_SF_MMA) *bytes = (size_t)sf_mma_bytes(rows, cols);
  else return NVFP4_ERR_INVALID_ARG;
  return NVFP4_OK;
}

nvfp4_status nvfp4_quantize(const void* x, int32_t xt, int64_t rows, int64_t cols, int64_t ldx,
                            const float* gscale_in, const nvfp4_tensor* out, float* amax_out,
                            nvfp4_stream_t stream) {
  if ((!x && rows > 0) || !valid_dtype(xt)) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_tensor(out);
  if (st != NVFP4_OK) return st;
  if (out->rows != rows || out->cols != cols || (rows > 0 && ldx < cols)) return NVFP4_ERR_SHAPE;
  if (!gscale_in && !amax_out) return NVFP4_ERR_INVALID_ARG;
  const int64_t esz = xt == NVFP4_BF16 ? 2 : 4;
  if (rows > 0 && (!aligned16(x) || (ldx * esz) % 16 != 0)) return NVFP4_ERR_ALIGNMENT;
  if ((amax_out && (reinterpret_cast<uintptr_t>(amax_out) & 3u)) ||
      (gscale_in && (reinterpret_cast<uintptr_t>(gscale_in) & 3u)))
    return NVFP4_ERR_ALIGNMENT;
  if (rows * cols * esz / 16 >= kMaxBlocks) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  nvfp4::QuantizeArgs a;
  a.x = x;
  a.x_bf16 = xt == NVFP4_BF16;
  a.rows = rows;
  a.cols = cols;
  a.ldx = ldx;
  a.gscale_in = gscale_in;
  a.codes = out->codes;
  a.ld_codes = out->ld_codes;
  a.scales = out->scales;
  a.ld_scales = out->ld_scales;
  a.sf_mma = out->sf_layout == NVFP4_SF_MMA;
  a.gscale_out = out->gscale;
  a.amax_out = amax_out;
  a.status = status;
  return cuda_status(nvfp4::launch_quantize(a, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_amax(const void* x, int32_t xt, int64_t rows, int64_t cols, int64_t ldx, float* amax_out,
                        nvfp4_stream_t stream) {
  if ((!x && rows > 0) || !amax_out || !valid_dtype(xt)) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || cols % 16 != 0 || (rows > 0 && ldx < cols)) return NVFP4_ERR_SHAPE;
  const int64_t esz = xt == NVFP4_BF16 ? 2 : 4;
  if (rows > 0 && (!aligned16(x) || (ldx * esz) % 16 != 0)) return NVFP4_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(amax_out) & 3u) return NVFP4_ERR_ALIGNMENT;
  if (rows * cols * esz / 16 >= kMaxBlocks) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  nvfp4_status st = current_device(&status);
  if (st != NVFP4_OK) return st;
  nvfp4::QuantizeArgs a = {};
  a.x = x;
  a.x_bf16 = xt == NVFP4_BF16;
  a.rows = rows;
  a.cols = cols;
  a.ldx = ldx;
  a.amax_out = amax_out;
  a.status = status;
  return cuda_status(nvfp4::launch_amax(a, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor* in, void* y, int32_t yt, int64_t ldy,
                              nvfp4_stream_t stream) {
  nvfp4_status st = check_tensor(in);
  if (st != NVFP4_OK) return st;
  if (!y || !valid_dtype(yt)) return NVFP4_ERR_INVALID_ARG;
  const int64_t esz = yt == NVFP4_BF16 ? 2 : 4;
  if (ldy < in->cols) return NVFP4_ERR_SHAPE;
  if (!aligned16(y) || (ldy * esz) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  nvfp4::DequantizeArgs a;
  a.codes = in->codes;
  a.ld_codes = in->ld_codes;
  a.scales = in->scales;
  a.ld_scales = in->ld_scales;
  a.sf_mma = in->sf_layout == NVFP4_SF_MMA;
  a.gscale = in->gscale;
  a.rows = in->rows;
  a.cols = in->cols;
  a.y = y;
  a.y_bf16 = yt == NVFP4_BF16;
  a.ldy = ldy;
  return cuda_status(nvfp4::launch_dequantize(a, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* W, void* C, int32_t ct,
                        int64_t ldc, const nvfp4_epilogue* ep, nvfp4_stream_t stream) {
  nvfp4_status st;
  if ((st = check_tensor(A)) != NVFP4_OK) return st;
  if ((st = check_tensor(W)) != NVFP4_OK) return st;
  if (A->sf_layout != NVFP4_SF_MMA || W->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
  if (A->cols != W->cols) return NVFP4_ERR_SHAPE;
  const int64_t M = A->rows, N = W->rows, K = A->cols;
  if (N % 16 != 0) return NVFP4_ERR_SHAPE;
  const bool fused = ep && ep->q_out;
  if (ep && (ep->act != NVFP4_ACT_NONE && ep->act != NVFP4_ACT_GELU_TANH)) return NVFP4_ERR_INVALID_ARG;
  if (ep && ep->reserved != 0) return NVFP4_ERR_INVALID_ARG;
  // at least one output: C, the requantized tensor, the activation dump or its amax
  const bool other_out = ep && (ep->q_out || ep->h_out || ep->q_amax_out);
  if (!C && !other_out) return NVFP4_ERR_INVALID_ARG;
  if (C) {
    if (!valid_dtype(ct)) return NVFP4_ERR_INVALID_ARG;
    const int64_t esz = ct == NVFP4_BF16 ? 2 : 4;
    if (ldc < N) return NVFP4_ERR_SHAPE;
    if (!aligned16(C) || (ldc * esz) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
  }
  if (fused) {
    if ((st = check_tensor(ep->q_out)) != NVFP4_OK) return st;
    if (ep->q_out->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
    if (ep->q_out->rows != M || ep->q_out->cols != N || N % 64 != 0) return NVFP4_ERR_SHAPE;
    if (!ep->q_gscale_in) return NVFP4_ERR_INVALID_ARG;
  }
  if (ep && ep->h_out && !aligned16(ep->h_out)) return NVFP4_ERR_ALIGNMENT;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  nvfp4::GemmArgs g;
  g.a = {A->codes, A->ld_codes, A->scales, A->gscale};
  g.w = {W->codes, W->ld_codes, W->scales, W->gscale};
  g.M = M;
  g.N = N;
  g.K = K;
  g.c = C;
  g.c_bf16 = ct == NVFP4_BF16;
  g.ldc = ldc;
  g.act = ep ? ep->act : 0;
  g.q_codes = fused ? ep->q_out->codes : nullptr;
  g.q_ld_codes = fused ? ep->q_out->ld_codes : 0;
  g.q_scales = fused ? ep->q_out->scales : nullptr;
  g.q_gscale_in = fused ? ep->q_gscale_in : nullptr;
  g.q_gscale_out = fused ? ep->q_out->gscale : nullptr;
  g.q_amax_out = ep ? ep->q_amax_out : nullptr;
  g.h_out = ep ? ep->h_out : nullptr;
  g.status = status;
  return cuda_status(nvfp4::launch_gemm(g, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------- KV cache

static int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

static nvfp4_status kv_geometry(int32_t heads, int32_t head_dim, int64_t chunk_tokens,
                                int32_t max_chunks, nvfp4::KVLayout* L, size_t* total) {
  if (heads <= 0 || head_dim <= 0 || head_dim % 16 != 0 || chunk_tokens <= 0 || max_chunks <= 0)
    return NVFP4_ERR_SHAPE;
  if (chunk_tokens > (1 << 24)) return NVFP4_ERR_SHAPE;
  const int64_t C = (int64_t)heads * head_dim;
  if (chunk_tokens * C / 16 * 64 >= kMaxBlocks) return NVFP4_ERR_SHAPE;
  const int64_t codes = chunk_tokens * C / 2, scales = chunk_tokens * C / 16;
  int64_t o = 0;
  L->heads = heads;
  L->head_dim = head_dim;
  L->chunk_tokens = chunk_tokens;
  L->max_chunks = max_chunks;
  L->slot_codes_bytes = codes;
  L->slot_scales_bytes = scales;
  L->off_k_codes = o;  o += align256(codes * max_chunks);
  L->off_v_codes = o;  o += align256(codes * max_chunks);
  L->off_k_scales = o; o += align256(scales * max_chunks);
  L->off_v_scales = o; o += align256(scales * max_chunks);
  L->off_mu = o;       o += align256(C * 4 * (int64_t)max_chunks);
  L->off_gscale = o;   o += align256(8 * (int64_t)max_chunks);
  L->off_tokens = o;   o += align256(4 * (int64_t)max_chunks);
  L->off_scratch = o;  o += align256(nvfp4::kv_scratch_bytes(heads, head_dim, chunk_tokens));
  *total = (size_t)o;
  return NVFP4_OK;
}

nvfp4_status nvfp4_kv_cache_bytes(int32_t heads, int32_t head_dim, int64_t chunk_tokens,
                                  int32_t max_chunks, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARG;
  nvfp4::KVLayout L;
  return kv_geometry(heads, head_dim, chunk_tokens, max_chunks, &L, bytes);
}

nvfp4_status nvfp4_kv_cache_init(void* dev_mem, size_t bytes, int32_t heads, int32_t head_dim,
                                 int64_t chunk_tokens, int32_t max_chunks, nvfp4_kv_cache* cache) {
  if (!dev_mem || !cache) return NVFP4_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_mem) & 255u) return NVFP4_ERR_ALIGNMENT;
  nvfp4::KVLayout L;
  size_t need = 0;
  nvfp4_status st = kv_geometry(heads, head_dim, chunk_tokens, max_chunks, &L, &need);
  if (st != NVFP4_OK) return st;
  // an allocation that ends before the append scratch serves kv_quant_append_noalloc
  // and the window calls; kv_quant_append then returns INVALID_ARG
  if (bytes < (size_t)L.off_scratch) return NVFP4_ERR_SHAPE;
  cache->base = static_cast<uint8_t*>(dev_mem);
  cache->bytes = bytes;
  cache->heads = heads;
  cache->head_dim = head_dim;
  cache->chunk_tokens = chunk_tokens;
  cache->max_chunks = max_chunks;
  cache->reserved = 0;
  cache->off_k_codes = L.off_k_codes;
  cache->off_v_codes = L.off_v_codes;
  cache->off_k_scales = L.off_k_scales;
  cache->off_v_scales = L.off_v_scales;
  cache->off_mu = L.off_mu;
  cache->off_gscale = L.off_gscale;
  cache->off_tokens = L.off_tokens;
  cache->off_scratch = L.off_scratch;
  cache->slot_codes_bytes = L.slot_codes_bytes;
  cache->slot_scales_bytes = L.slot_scales_bytes;
  return NVFP4_OK;
}

// Re-derives the layout from the geometry and checks it against the handle.  A
// caller that never uses the cache's append scratch (kv_quant_append_noalloc) may
// hand over an allocation that ends where the scratch region would begin.
static nvfp4_status check_cache(const nvfp4_kv_cache* c, nvfp4::KVLayout* L, bool needs_scratch = true) {
  if (!c || !c->base) return NVFP4_ERR_INVALID_ARG;
  size_t need = 0;
  nvfp4_status st = kv_geometry(c->heads, c->head_dim, c->chunk_tokens, c->max_chunks, L, &need);
  if (st != NVFP4_OK) return st;
  if (!needs_scratch) need = (size_t)L->off_scratch;
  if (c->bytes < need || L->off_scratch != c->off_scratch || L->off_mu != c->off_mu ||
      L->off_tokens != c->off_tokens)
    return NVFP4_ERR_INVALID_ARG;
  L->base = c->base;
  return NVFP4_OK;
}

nvfp4_status kv_quant_append(const nvfp4_kv_cache* cache, const void* k, const void* v,
                             int64_t tokens, int32_t slot, nvfp4_stream_t stream) {
  nvfp4::KVLayout L;
  nvfp4_status st = check_cache(cache, &L);
  if (st != NVFP4_OK) return st;
  if (!k || !v) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return NVFP4_ERR_ALIGNMENT;
  if (tokens < 1 || tokens > cache->chunk_tokens) return NVFP4_ERR_SHAPE;
  if (slot < 0 || slot >= cache->max_chunks) return NVFP4_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_kv_append(L, k, v, tokens, slot, status,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status kv_quant_append_noalloc(const nvfp4_kv_cache* cache, const void* k, const void* v,
                                     int64_t tokens, int32_t slot, nvfp4_stream_t stream) {
  nvfp4::KVLayout L;
  nvfp4_status st = check_cache(cache, &L, /*needs_scratch=*/false);
  if (st != NVFP4_OK) return st;
  if (!k || !v) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return NVFP4_ERR_ALIGNMENT;
  if (tokens < 1 || tokens > cache->chunk_tokens) return NVFP4_ERR_SHAPE;
  if (slot < 0 || slot >= cache->max_chunks) return NVFP4_ERR_INVALID_ARG;
  if ((int64_t)cache->heads * cache->head_dim > NVFP4_NOALLOC_MAX_COLUMNS) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_kv_append_noalloc(L, k, v, tokens, slot, status,
                                                     reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status kv_dequant_window_tokens(const nvfp4_kv_cache* cache, const int32_t* slots_host,
                                      const int32_t* tokens_host, int32_t n_slots, void* k_out,
                                      void* v_out, nvfp4_stream_t stream) {
  nvfp4::KVLayout L;
  nvfp4_status st = check_cache(cache, &L, /*needs_scratch=*/false);
  if (st != NVFP4_OK) return st;
  if (!slots_host || !tokens_host || !k_out || !v_out) return NVFP4_ERR_INVALID_ARG;
  if (n_slots < 1 || n_slots > nvfp4::kMaxWindowSlots) return NVFP4_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int i = 0; i < n_slots; ++i) {
    if (slots_host[i] < 0 || slots_host[i] >= cache->max_chunks) return NVFP4_ERR_INVALID_ARG;
    if (tokens_host[i] < 1 || tokens_host[i] > cache->chunk_tokens) return NVFP4_ERR_SHAPE;
    total += tokens_host[i];
  }
  if (!aligned16(k_out) || !aligned16(v_out)) return NVFP4_ERR_ALIGNMENT;
  const int64_t C = (int64_t)cache->heads * cache->head_dim;
  if (total * C / 16 >= kMaxBlocks) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  if ((st = current_device(&status)) != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_kv_window(L, slots_host, tokens_host, n_slots, k_out, v_out, status,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status kv_window_scores(const nvfp4_kv_cache* cache, const int32_t* slots_host, const int32_t* tokens_host,
                              int32_t n_slots, const void* q, int64_t tq, int64_t ldq, float scale, void* s_out,
                              int32_t st, int64_t ld_s, nvfp4_stream_t stream) {
  nvfp4::KVLayout L;
  nvfp4_status st_ = check_cache(cache, &L, /*needs_scratch=*/false);
  if (st_ != NVFP4_OK) return st_;
  if (!slots_host || !tokens_host || !s_out || (!q && tq > 0) || !valid_dtype(st)) return NVFP4_ERR_INVALID_ARG;
  if (n_slots < 1 || n_slots > nvfp4::kMaxWindowSlots) return NVFP4_ERR_INVALID_ARG;
  if (cache->head_dim != 128) return NVFP4_ERR_SHAPE;
  int64_t total = 0;
  for (int i = 0; i < n_slots; ++i) {
    if (slots_host[i] < 0 || slots_host[i] >= cache->max_chunks) return NVFP4_ERR_INVALID_ARG;
    if (tokens_host[i] < 1 || tokens_host[i] > cache->chunk_tokens) return NVFP4_ERR_SHAPE;
    total += tokens_host[i];
  }
  const int64_t esz = st == NVFP4_BF16 ? 2 : 4;
  if (tq < 0 || ldq < (int64_t)cache->heads * 128 || ld_s < total) return NVFP4_ERR_SHAPE;
  if (tq > (1ll << 31) || total > (1ll << 31) || (int64_t)cache->heads > 65535) return NVFP4_ERR_SHAPE;
  if (tq > 0 && (!aligned16(q) || (ldq * 2) % 16 != 0)) return NVFP4_ERR_ALIGNMENT;
  if (!aligned16(s_out) || (ld_s * esz) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
  if (!(scale == scale) || scale > 3.402823466e38f || scale < -3.402823466e38f) return NVFP4_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  if ((st_ = current_device(&status)) != NVFP4_OK) return st_;
  return cuda_status(nvfp4::launch_kv_scores(L, slots_host, tokens_host, n_slots, q, tq, ldq, scale, s_out,
                                             st == NVFP4_BF16, ld_s, status,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status kv_window_context(const nvfp4_kv_cache* cache, const int32_t* slots_host, const int32_t* tokens_host,
                               int32_t n_slots, const void* p, int64_t tq, int64_t ld_p, void* o_out, int32_t ot,
                               int64_t ldo, nvfp4_stream_t stream) {
  nvfp4::KVLayout L;
  nvfp4_status st_ = check_cache(cache, &L, /*needs_scratch=*/false);
  if (st_ != NVFP4_OK) return st_;
  if (!slots_host || !tokens_host || !o_out || (!p && tq > 0) || !valid_dtype(ot)) return NVFP4_ERR_INVALID_ARG;
  if (n_slots < 1 || n_slots > nvfp4::kMaxWindowSlots) return NVFP4_ERR_INVALID_ARG;
  if (cache->head_dim != 128) return NVFP4_ERR_SHAPE;
  int64_t total = 0;
  for (int i = 0; i < n_slots; ++i) {
    if (slots_host[i] < 0 || slots_host[i] >= cache->max_chunks) return NVFP4_ERR_INVALID_ARG;
    if (tokens_host[i] < 1 || tokens_host[i] > cache->chunk_tokens) return NVFP4_ERR_SHAPE;
    total += tokens_host[i];
  }
  const int64_t esz = ot == NVFP4_BF16 ? 2 : 4;
  if (tq < 0 || ld_p < total || ldo < (int64_t)cache->heads * 128) return NVFP4_ERR_SHAPE;
  // at most 65535 query groups of up to 4 query tiles of 128
  if (tq > 65535ll * 4 * 128 || total > (1ll << 31) || (int64_t)cache->heads > 65535) return NVFP4_ERR_SHAPE;
  if (tq > 0 && (!aligned16(p) || (ld_p * 2) % 16 != 0)) return NVFP4_ERR_ALIGNMENT;
  if (!aligned16(o_out) || (ldo * esz) % 16 != 0) return NVFP4_ERR_ALIGNMENT;
  unsigned* status = nullptr;
  if ((st_ = current_device(&status)) != NVFP4_OK) return st_;
  return cuda_status(nvfp4::launch_kv_context(L, slots_host, tokens_host, n_slots, p, tq, ld_p, o_out,
                                              ot == NVFP4_BF16, ldo, status, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status kv_dequant_window(const nvfp4_kv_cache* cache, const int32_t* slots_host,
                               int32_t n_slots, void* k_out, void* v_out, nvfp4_stream_t stream) {
  if (!cache || n_slots < 1 || n_slots > nvfp4::kMaxWindowSlots) return NVFP4_ERR_INVALID_ARG;
  if (cache->chunk_tokens > (1 << 24)) return NVFP4_ERR_SHAPE;
  int32_t tokens[nvfp4::kMaxWindowSlots];
  for (int i = 0; i < n_slots; ++i) tokens[i] = (int32_t)cache->chunk_tokens;
  return kv_dequant_window_tokens(cache, slots_host, tokens, n_slots, k_out, v_out, stream);
}

nvfp4_status nvfp4_lora_merge(const void* w, nvfp4_dtype wt, int64_t rows, int64_t cols, int64_t ldw,
                              const float* lora_b, const float* lora_a, int32_t rank, float scale,
                              float* out, int64_t ldo, nvfp4_stream_t stream) {
  if (!valid_dtype(wt) || rank < 1 || rank > 4096) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!w || !lora_b || !lora_a || !out) return NVFP4_ERR_INVALID_ARG;
  if (ldw < cols || ldo < cols) return NVFP4_ERR_SHAPE;
  if (rows > (int64_t)1 << 31 || cols > (int64_t)1 << 31) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  nvfp4_status st = current_device(&status);
  if (st != NVFP4_OK) return st;
  nvfp4::LoraArgs a;
  a.w = w;
  a.w_bf16 = wt == NVFP4_BF16;
  a.rows = rows;
  a.cols = cols;
  a.ldw = ldw;
  a.b = lora_b;
  a.a = lora_a;
  a.rank = rank;
  a.scale = scale;
  a.out = out;
  a.ldo = ldo;
  return cuda_status(nvfp4::launch_lora_merge(a, reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_amax_history_push(float* history, int32_t len, const float* amax_new, float* gscale_out,
                                     nvfp4_stream_t stream) {
  if (!history || !amax_new || !gscale_out) return NVFP4_ERR_INVALID_ARG;
  if (len < 1 || len > nvfp4::kMaxHistory) return NVFP4_ERR_SHAPE;
  unsigned* status = nullptr;
  nvfp4_status st = current_device(&status);
  if (st != NVFP4_OK) return st;
  return cuda_status(nvfp4::launch_amax_history(history, len, amax_new, gscale_out, status,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_debug_grid_barrier(uint32_t extra_arrivals, uint64_t wait_limit_ns) {
  nvfp4::grid_barrier_debug(extra_arrivals, (unsigned long long)wait_limit_ns);
  return NVFP4_OK;
}

nvfp4_status nvfp4_debug_gemm_fault(int32_t drop_first_stage, uint64_t wait_limit_ns) {
  nvfp4::gemm_debug_fault(drop_first_stage, (unsigned long long)wait_limit_ns);
  return NVFP4_OK;
}

nvfp4_status nvfp4_get_device_status(int32_t device, int32_t* status_out, int32_t clear) {
  if (!status_out) return NVFP4_ERR_INVALID_ARG;
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaSetDevice(device) != cudaSuccess) return NVFP4_ERR_INVALID_ARG;
  unsigned* status = nullptr;
  nvfp4_status st = init_device(device, &status);
  if (st == NVFP4_OK) {
    unsigned v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
      st = NVFP4_ERR_CUDA;
    else {
      *status_out = (int32_t)v;
      if (clear && cudaMemset(status, 0, sizeof(unsigned)) != cudaSuccess) st = NVFP4_ERR_CUDA;
      if (clear && cudaDeviceSynchronize() != cudaSuccess) st = NVFP4_ERR_CUDA;
    }
  }
  cudaSetDevice(prev);
  return st;
}

}  // extern "C"
