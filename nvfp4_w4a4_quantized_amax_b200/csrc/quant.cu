// quant.cu — NVFP4 activation quantization and dequantization (HBM-bound).
//
// techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存", §一:
// every 16 values share one FP8 scale and the whole tensor shares one FP32 scale.
// The tensor scale needs max|x| before any block can be encoded, so quantization
// with an unknown scale is two passes over x: amax_kernel, then encode_kernel.
// With a supplied scale (one pass) encode_kernel also reports max|x| for the
// caller's next calibration.
//
// Memory traffic per element (bf16 in): amax pass 2 B read; encode pass 2 B read,
// 0.5 B codes + 1/16 B scale written.  Loads are 128-bit and read-only-path.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;
constexpr int kDequantBatch = 2;  // half-blocks per thread and pass of the dequantize kernel (1, 2, 4, 8 measured: 2)

__device__ __forceinline__ void block_max_atomic(unsigned v, unsigned* dst) {
  __shared__ unsigned red[kThreads / 32];
  v = warp_max_u32(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kThreads / 32 ? red[lane] : 0u;
    v = warp_max_u32(v);
    if (lane == 0 && v != 0u) atomicMax(dst, v);
  }
}

// max |x| as binary32 bits (non-negative floats order like unsigned integers; a
// NaN or Inf anywhere yields bits >= 0x7F800000).  x is read in 16-byte chunks,
// chunks_per_row per row.
template <bool kBf16>
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint8_t* __restrict__ x,
                                                        int64_t row_bytes, int64_t nchunks,
                                                        FastDiv cpr, unsigned* amax_bits) {
  pdl_trigger();
  pdl_wait();
  unsigned m = 0;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nchunks; i += stride) {
    const uint32_t r = cpr.div((uint32_t)i);
    const uint32_t c = (uint32_t)i - r * cpr.d;
    const uint4 v = ldg_nc_v4(x + (int64_t)r * row_bytes + (int64_t)c * 16);
    if (kBf16) {
      m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    } else {
      m = max(m, v.x & 0x7FFFFFFFu);
      m = max(m, v.y & 0x7FFFFFFFu);
      m = max(m, v.z & 0x7FFFFFFFu);
      m = max(m, v.w & 0x7FFFFFFFu);
    }
  }
  if (kBf16) m = max(m >> 16, m & 0xFFFFu) << 16;
  block_max_atomic(m, amax_bits);
}

struct EncodeParams {
  const uint8_t* x;
  int64_t x_row_bytes;
  uint8_t* codes;
  int64_t ld_codes;
  uint8_t* scales;
  int64_t ld_scales;
  int64_t groups;   // MMA layout: ceil(nb / 4)
  int64_t rows, nb; // real rows and blocks per row
  int64_t nvblocks; // blocks visited (includes MMA-layout padding)
  FastDiv vb_per_row;
  const float* gscale_in;
  const unsigned* amax_bits;
  float* gscale_out;
  unsigned* amax_accum;  // nullable (one-pass mode)
  unsigned* status;
};

// The 16 values of virtual block vb (16 bf16 = 32 bytes, or 16 FP32 = 64 bytes).
template <bool kBf16>
__device__ __forceinline__ void load_block(const EncodeParams& p, uint32_t r, uint32_t j, float (&v)[16]) {
  const uint8_t* src = p.x + (int64_t)r * p.x_row_bytes + (int64_t)j * (kBf16 ? 32 : 64);
  if (kBf16) {
    // the second load finds the other half of each 32-byte sector in L1
    const uint4 a = ldg_nc_v4_l1(src), b = ldg_nc_v4_l1(src + 16);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[2 * k] = bf16_lo(w[k]);
      v[2 * k + 1] = bf16_hi(w[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 a = ldg_nc_v4_l1(src + 16 * k);
      v[4 * k] = __uint_as_float(a.x);
      v[4 * k + 1] = __uint_as_float(a.y);
      v[4 * k + 2] = __uint_as_float(a.z);
      v[4 * k + 3] = __uint_as_float(a.w);
    }
  }
}

// Encodes virtual block vb with tensor scale g (d6 = RN(6 g), r6 = RN(1 / d6)):
// block amax -> E4M3 scale -> 16 codes.  Padding blocks of the tensor-core layout
// get a zero scale.  local_max accumulates max|x| bits when `track` is set.
template <bool kBf16, bool kMma>
__device__ __forceinline__ void encode_block(const EncodeParams& p, int64_t vb, float g, float d6, float r6,
                                             bool track, unsigned& local_max) {
  const uint32_t r = p.vb_per_row.div((uint32_t)vb);
  const uint32_t j = (uint32_t)vb - r * p.vb_per_row.d;
  const int64_t soff = kMma ? sf_mma_offset(r, j, p.groups) : (int64_t)r * p.ld_scales + j;
  if (kMma && (r >= p.rows || j >= p.nb)) {  // padding of the tensor-core layout
    p.scales[soff] = 0;
    return;
  }
  float v[16];
  load_block<kBf16>(p, r, j, v);
  float amax_b = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax_b = fmaxf(amax_b, fabsf(v[k]));
  if (track) {
    unsigned bits = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) bits = max(bits, __float_as_uint(v[k]) & 0x7FFFFFFFu);
    local_max = max(local_max, bits);
  }
  const uint32_t s = block_scale_fast(amax_b, d6, r6);
  const BlockEncoder enc(e4m3_to_float(s) * g);
  float v0[8], v1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v0[k] = v[k];
    v1[k] = v[8 + k];
  }
  uint2 out;
  out.x = enc.encode8s(v0);
  out.y = enc.encode8s(v1);
  stg_v2(p.codes + (int64_t)r * p.ld_codes + (int64_t)j * 8, out);
  p.scales[soff] = (uint8_t)s;
}

// One thread encodes one 16-value block: block amax -> E4M3 scale -> 16 codes.  Six
// resident CTAs per SM (40 registers, no spills): the pass is issue-bound, and 6
// against 4 CTAs measured 3 % faster on 32768x3072 and 8192x14336 (7 and 8 spill).
template <bool kBf16, bool kMma>
__global__ void __launch_bounds__(kThreads, 6) encode_kernel(EncodeParams p) {
  pdl_trigger();
  pdl_wait();
  float g;
  if (p.gscale_in) {
    g = *p.gscale_in;
    if (!(g >= 0.0f) || !(g <= 3.402823466e38f)) {
      if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, kStatusNonfinite);
      return;
    }
  } else {
    const unsigned ab = *p.amax_bits;
    if (ab >= 0x7F800000u) {
      if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, kStatusNonfinite);
      return;
    }
    g = __uint_as_float(ab) / 2688.0f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.gscale_out = g;
  const float d6 = 6.0f * g;
  const float r6 = 1.0f / d6;

  unsigned local_max = 0;
  const bool track = p.amax_accum != nullptr;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  // Blocks are visited from the end of x backwards: the amax pass read x front to
  // back, so its most recent reads (still in L2) are encoded first.
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < p.nvblocks; i += stride)
    encode_block<kBf16, kMma>(p, p.nvblocks - 1 - i, g, d6, r6, track, local_max);
  if (track) {
    if (local_max >= 0x7F800000u) set_status(p.status, kStatusNonfinite);
    block_max_atomic(local_max, p.amax_accum);
  }
}

// Grid-barrier counters of quantize_fused_kernel, one per launch slot: launches take
// slots round robin and zero theirs on the stream first, so a slot is reused only
// after kGridSyncSlots later launches (calls on other streams that overlap that many
// launches would share a counter).
constexpr int kGridSyncSlots = 256;
__device__ unsigned g_grid_sync[kGridSyncSlots];

// Quantization with an unknown tensor scale in ONE launch, for a tensor small
// enough to stay in L2 between its two reads: every CTA takes max|x| over a
// grid-stride share of x, the grid meets at a bounded barrier (all CTAs of the
// one-wave grid are resident), then every CTA encodes its blocks with
// g = RN(amax / 2688) while x is still in L2.  Replaces the zero + amax + encode
// chain (two dependent launch boundaries) for such tensors; the result is the same
// bits.  g_grid_sync[slot] is the grid-barrier counter, zeroed on the stream before
// the launch.  The kernel lets its dependents start only once the whole grid has
// met, so a dependent grid can never hold resources that one of its CTAs still needs.
template <bool kBf16, bool kMma>
__global__ void __launch_bounds__(kThreads) quantize_fused_kernel(EncodeParams p, unsigned* amax_bits,
                                                                  int slot, int64_t nchunks, FastDiv cpr,
                                                                  unsigned barrier_extra,
                                                                  unsigned long long barrier_limit_ns) {
  pdl_wait();
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  const int64_t first = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  // first pass: max|x| with one coalesced 16-byte load per thread and step (the
  // layout of the amax kernel); x lands in L2 for the second pass
  unsigned m = 0;
  for (int64_t i = first; i < nchunks; i += stride) {
    const uint32_t r = cpr.div((uint32_t)i);
    const uint32_t c = (uint32_t)i - r * cpr.d;
    const uint4 v = ldg_nc_v4(p.x + (int64_t)r * p.x_row_bytes + (int64_t)c * 16);
    if (kBf16) {
      m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
      m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
    } else {
      m = max(m, v.x & 0x7FFFFFFFu);
      m = max(m, v.y & 0x7FFFFFFFu);
      m = max(m, v.z & 0x7FFFFFFFu);
      m = max(m, v.w & 0x7FFFFFFFu);
    }
  }
  if (kBf16) m = max(m >> 16, m & 0xFFFFu) << 16;
  block_max_atomic(m, amax_bits);
  if (!grid_barrier_n(&g_grid_sync[slot], gridDim.x + barrier_extra, barrier_limit_ns)) {
    if (threadIdx.x == 0) set_status(p.status, kStatusTimeout);
    pdl_trigger();
    return;
  }
  pdl_trigger();  // the whole grid is resident and past its first pass
  const unsigned ab = ld_relaxed_gpu(amax_bits);
  if (ab >= 0x7F800000u) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, kStatusNonfinite);
    return;
  }
  const float g = __uint_as_float(ab) / 2688.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.gscale_out = g;
  const float d6 = 6.0f * g;
  const float r6 = 1.0f / d6;
  unsigned unused = 0;
  // second pass from the end backwards: the first pass's latest reads are the most
  // likely still in L2
  for (int64_t i = first; i < p.nvblocks; i += stride)
    encode_block<kBf16, kMma>(p, p.nvblocks - 1 - i, g, d6, r6, false, unused);
}

struct DequantParams {
  const uint8_t* codes;
  int64_t ld_codes;
  const uint8_t* scales;
  int64_t ld_scales;
  int64_t groups;
  const float* gscale;
  int64_t nblocks;
  FastDiv nb_per_row;
  uint8_t* y;
  int64_t y_row_bytes;
};

// Two threads per 16-value block (8 values each): y = RN(RN(e2m1 * s) * g).  A
// warp reads 128 contiguous bytes of codes and writes 512 contiguous bytes of bf16.
template <bool kMma, bool kBf16Out>
__global__ void __launch_bounds__(kThreads) dequant_kernel(DequantParams p) {
  pdl_trigger();
  pdl_wait();
  const float g = *p.gscale;
  const int64_t total = 2 * p.nblocks;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  // kDequantBatch half-blocks per thread and pass, their code words and scale bytes
  // all loaded before the first is decoded: the reads are small next to the writes,
  // and one load in flight per thread leaves the loop waiting on DRAM latency
  for (int64_t hb0 = (int64_t)blockIdx.x * kThreads + threadIdx.x; hb0 < total; hb0 += kDequantBatch * stride) {
    uint32_t c[kDequantBatch], sb[kDequantBatch], rr[kDequantBatch], jj[kDequantBatch];
#pragma unroll
    for (int u = 0; u < kDequantBatch; ++u) {
      const int64_t hb = hb0 + u * stride;
      c[u] = 0;
      sb[u] = 0;
      rr[u] = jj[u] = 0;
      if (hb < total) {
        const uint32_t b = (uint32_t)(hb >> 1);
        const uint32_t r = p.nb_per_row.div(b);
        const uint32_t j = b - r * p.nb_per_row.d;
        c[u] = *reinterpret_cast<const uint32_t*>(p.codes + (int64_t)r * p.ld_codes + (int64_t)j * 8 + (hb & 1) * 4);
        sb[u] = p.scales[kMma ? sf_mma_offset(r, j, p.groups) : (int64_t)r * p.ld_scales + j];
        rr[u] = r;
        jj[u] = j;
      }
    }
#pragma unroll
    for (int u = 0; u < kDequantBatch; ++u) {
      const int64_t hb = hb0 + u * stride;
      if (hb >= total) break;
      const int half = (int)(hb & 1);
      uint32_t h[4];
      e2m1x8_times_scale(c[u], e4m3_to_f16x2_bcast(sb[u]), h);
      float y[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        f16x2_to_f32x2(h[k], y[2 * k], y[2 * k + 1]);  // e2m1 * s, exact
        y[2 * k] *= g;
        y[2 * k + 1] *= g;
      }
      uint8_t* dst = p.y + (int64_t)rr[u] * p.y_row_bytes + (int64_t)jj[u] * (kBf16Out ? 32 : 64) +
                     half * (kBf16Out ? 16 : 32);
      if (kBf16Out) {
        stg_v4(dst, make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                               pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7])));
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k)
          stg_v4(dst + 16 * k, make_uint4(__float_as_uint(y[4 * k]), __float_as_uint(y[4 * k + 1]),
                                          __float_as_uint(y[4 * k + 2]), __float_as_uint(y[4 * k + 3])));
      }
    }
  }
}


__global__ void zero_sync_kernel(unsigned* amax_bits, int slot) {
  pdl_wait();
  if (threadIdx.x == 0) *amax_bits = 0u;
  if (threadIdx.x == 1) g_grid_sync[slot] = 0u;
}

// Zeroes n words before an accumulation: a kernel rather than a memset, so that
// its launch overlaps the previous kernel.  It does not trigger its dependents
// early: the kernel after it starts only once it is done (as after a memset).
__global__ void zero_words_kernel(unsigned* p, int n) {
  pdl_wait();
  for (int i = threadIdx.x; i < n; i += blockDim.x) p[i] = 0u;
}

// Amax history of a requantizing epilogue (newest first): shift in *amax_new and
// write g = RN(max(history) / 2688).  One CTA; a non-finite value changes nothing.
constexpr int kHistThreads = 256;
__global__ void __launch_bounds__(kHistThreads) amax_history_kernel(float* history, int len, const float* amax_new,
                                                                   float* g_out, unsigned* status) {
  pdl_trigger();
  pdl_wait();
  __shared__ float old[kMaxHistory];
  __shared__ unsigned red[kHistThreads / 32];
  const float a = *amax_new;
  if (!(fabsf(a) <= 3.402823466e38f)) {
    if (threadIdx.x == 0) set_status(status, kStatusNonfinite);
    return;
  }
  for (int i = threadIdx.x; i < len; i += kHistThreads) old[i] = history[i];
  __syncthreads();
  unsigned m = 0;  // max of non-negative floats as ordered bits
  for (int i = threadIdx.x; i < len; i += kHistThreads) {
    const float v = i == 0 ? a : old[i - 1];
    history[i] = v;
    m = max(m, __float_as_uint(fmaxf(v, 0.0f)));
  }
  m = warp_max_u32(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned mm = 0;
    for (int w = 0; w < kHistThreads / 32; ++w) mm = max(mm, red[w]);
    *g_out = __uint_as_float(mm) / 2688.0f;
  }
}

}  // namespace

// The amax pass alone: max|x| as binary32 bits into amax_bits (zeroed first).
static cudaError_t launch_amax_pass(const void* x, bool x_bf16, int64_t rows, int64_t cols, int64_t ldx,
                                    unsigned* amax_bits, cudaStream_t s) {
  const int64_t esz = x_bf16 ? 2 : 4;
  const int64_t cpr = cols * esz / 16;
  const int64_t n = rows * cpr;
  if (x_bf16)
    launch_pdl(amax_kernel<true>, wave_grid<amax_kernel<true>>(kThreads, n), kThreads, 0, s, (const uint8_t*)x,
               ldx * esz, n, FastDiv((uint32_t)cpr), amax_bits);
  else
    launch_pdl(amax_kernel<false>, wave_grid<amax_kernel<false>>(kThreads, n), kThreads, 0, s, (const uint8_t*)x,
               ldx * esz, n, FastDiv((uint32_t)cpr), amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_amax(const QuantizeArgs& a, cudaStream_t s) {
  cudaError_t e = launch_zero_words(a.amax_out, 1, s);
  if (e != cudaSuccess || a.rows == 0) return e;
  return launch_amax_pass(a.x, a.x_bf16, a.rows, a.cols, a.ldx, reinterpret_cast<unsigned*>(a.amax_out), s);
}

// Tensors up to this many bytes take the one-launch quantization (two reads of x
// that stay in the 126 MB L2 between them; half of L2 leaves room for the outputs
// and for what other kernels keep there).
constexpr int64_t kFusedQuantizeMaxBytes = 64ll << 20;

template <bool kBf16, bool kMma>
static cudaError_t launch_fused(const EncodeParams& p, unsigned* amax_bits, cudaStream_t s) {
  static std::atomic<unsigned> next_slot{0};
  const int slot = (int)(next_slot.fetch_add(1, std::memory_order_relaxed) % kGridSyncSlots);
  launch_pdl(zero_sync_kernel, 1, 32, 0, s, amax_bits, slot);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // one wave: every CTA is resident at once, which the grid barrier needs
  const int grid = wave_grid<quantize_fused_kernel<kBf16, kMma>>(kThreads, p.nvblocks);
  const int64_t cpr = p.nb * (kBf16 ? 2 : 4);  // 16-byte chunks of x per row
  launch_pdl(quantize_fused_kernel<kBf16, kMma>, grid, kThreads, 0, s, p, amax_bits, slot, p.rows * cpr,
             FastDiv((uint32_t)cpr), grid_barrier_extra(), grid_barrier_limit_ns());
  return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantizeArgs& a, cudaStream_t s) {
  const int64_t esz = a.x_bf16 ? 2 : 4;
  const int64_t nb = a.cols / 16;
  unsigned* amax_bits = reinterpret_cast<unsigned*>(a.amax_out);
  const bool fused = !a.gscale_in && a.rows > 0 && a.rows * a.ldx * esz <= kFusedQuantizeMaxBytes;
  if (a.amax_out && !fused) {
    cudaError_t e = launch_zero_words(a.amax_out, 1, s);
    if (e != cudaSuccess) return e;
  }
  if (a.rows == 0) {
    if (!a.gscale_in) {  // empty tensor: amax = 0, g = 0
      return cudaMemsetAsync(a.gscale_out, 0, sizeof(float), s);
    }
    return cudaMemcpyAsync(a.gscale_out, a.gscale_in, sizeof(float), cudaMemcpyDeviceToDevice, s);
  }
  if (!a.gscale_in && !fused) {
    cudaError_t e = launch_amax_pass(a.x, a.x_bf16, a.rows, a.cols, a.ldx, amax_bits, s);
    if (e != cudaSuccess) return e;
  }
  EncodeParams p;
  p.x = (const uint8_t*)a.x;
  p.x_row_bytes = a.ldx * esz;
  p.codes = a.codes;
  p.ld_codes = a.ld_codes;
  p.scales = a.scales;
  p.ld_scales = a.ld_scales;
  p.groups = (nb + 3) / 4;
  p.rows = a.rows;
  p.nb = nb;
  const int64_t vb_per_row = a.sf_mma ? p.groups * 4 : nb;
  const int64_t vrows = a.sf_mma ? (a.rows + 127) / 128 * 128 : a.rows;
  p.nvblocks = vrows * vb_per_row;
  p.vb_per_row = FastDiv((uint32_t)vb_per_row);
  p.gscale_in = a.gscale_in;
  p.amax_bits = amax_bits;
  p.gscale_out = a.gscale_out;
  p.amax_accum = a.gscale_in ? amax_bits : nullptr;
  p.status = a.status;
  if (fused) {
    if (a.x_bf16) return a.sf_mma ? launch_fused<true, true>(p, amax_bits, s) : launch_fused<true, false>(p, amax_bits, s);
    return a.sf_mma ? launch_fused<false, true>(p, amax_bits, s) : launch_fused<false, false>(p, amax_bits, s);
  }
  const int64_t n = p.nvblocks;
  if (a.x_bf16) {
    if (a.sf_mma) launch_pdl(encode_kernel<true, true>, wave_grid<encode_kernel<true, true>>(kThreads, n), kThreads, 0, s, p);
    else launch_pdl(encode_kernel<true, false>, wave_grid<encode_kernel<true, false>>(kThreads, n), kThreads, 0, s, p);
  } else {
    if (a.sf_mma) launch_pdl(encode_kernel<false, true>, wave_grid<encode_kernel<false, true>>(kThreads, n), kThreads, 0, s, p);
    else launch_pdl(encode_kernel<false, false>, wave_grid<encode_kernel<false, false>>(kThreads, n), kThreads, 0, s, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const DequantizeArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  DequantParams p;
  p.codes = a.codes;
  p.ld_codes = a.ld_codes;
  p.scales = a.scales;
  p.ld_scales = a.ld_scales;
  const int64_t nb = a.cols / 16;
  p.groups = (nb + 3) / 4;
  p.gscale = a.gscale;
  p.nblocks = a.rows * nb;
  p.nb_per_row = FastDiv((uint32_t)nb);
  p.y = (uint8_t*)a.y;
  p.y_row_bytes = a.ldy * (a.y_bf16 ? 2 : 4);
  const int64_t n = 2 * p.nblocks;
  if (a.sf_mma) {
    if (a.y_bf16) launch_pdl(dequant_kernel<true, true>, wave_grid<dequant_kernel<true, true>>(kThreads, n), kThreads, 0, s, p);
    else launch_pdl(dequant_kernel<true, false>, wave_grid<dequant_kernel<true, false>>(kThreads, n), kThreads, 0, s, p);
  } else {
    if (a.y_bf16) launch_pdl(dequant_kernel<false, true>, wave_grid<dequant_kernel<false, true>>(kThreads, n), kThreads, 0, s, p);
    else launch_pdl(dequant_kernel<false, false>, wave_grid<dequant_kernel<false, false>>(kThreads, n), kThreads, 0, s, p);
  }
  return cudaGetLastError();
}

}  // namespace nvfp4

namespace nvfp4 {
namespace {
std::atomic<unsigned> g_barrier_extra{0};
std::atomic<unsigned long long> g_barrier_limit_ns{0};
}  // namespace

void grid_barrier_debug(unsigned extra, unsigned long long limit_ns) {
  g_barrier_extra.store(extra);
  g_barrier_limit_ns.store(limit_ns);
}
unsigned grid_barrier_extra() { return g_barrier_extra.load(); }
unsigned long long grid_barrier_limit_ns() {
  const unsigned long long v = g_barrier_limit_ns.load();
  return v ? v : kGridBarrierLimitNs;
}

cudaError_t launch_zero_words(void* p, int n_words, cudaStream_t s) {
  launch_pdl(zero_words_kernel, 1, 32, 0, s, static_cast<unsigned*>(p), n_words);
  return cudaGetLastError();
}

cudaError_t launch_amax_history(float* history, int len, const float* amax_new, float* g_out, unsigned* status,
                                cudaStream_t s) {
  launch_pdl(amax_history_kernel, 1, kHistThreads, 0, s, history, len, amax_new, g_out, status);
  return cudaGetLastError();
}
}  // namespace nvfp4
