// kv.cu — NVFP4 KV cache: quantize-on-append (in place) and multi-chunk window
// dequantization.
//
// techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存", §四:
// K gets a simple mean subtraction, then K and V are stored in NVFP4; a dedicated
// parallel CUDA kernel dequantizes several cache chunks of one window at once.
// github.zuobiaodaohang.com, "长视频生成的两堵物理墙", section "NVFP4：数据体积砍到 1/4":
// the quantized KV cache is updated in place.
//
// Reading fixed here: mu[h, d] = RN_f32(exact sum over the chunk's tokens / T),
// K' = RN(k - mu), one tensor scale per chunk for K' and one for V, blocks of 16
// along head_dim.  The exact sum makes mu independent of summation order.
//
// Append = 3 kernels on one stream:
//   kv_stats_kernel : per (token split, column) double partial sums, min, max,
//                     smallest nonzero |k|; max|v| (one read of K and V)
//   kv_mu_kernel    : per column: mu (exact; see below), max|K'| over the chunk
//   kv_encode_kernel: K' and V -> codes and scales of the slot (second read)
// The double partial sums are exact whenever a column's nonzero magnitudes span at
// most 45 - ceil(log2 T) binades (every value is then a multiple of the smallest
// value's last bit and no partial sum can exceed 53 bits); a column outside that
// range is summed exactly with integer limbs by kv_mu_kernel itself.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kStatsThreads = 256;   // 8 warps; each lane owns 8 consecutive columns
constexpr int kStatsCols = 256;      // columns per CTA
constexpr int kSplits = 64;          // most token splits of the stats pass (scratch size)
constexpr int kStatsUnroll = 2;      // token rows in flight per warp (2, 4, 6, 8 measured: 2 fastest)
constexpr int kMuThreads = 256;      // 8 warps share the splits of kMuCols columns
constexpr int kMuCols = 32;
constexpr int kEncThreads = 256;

// scratch layout (byte offsets from the scratch base)
struct Scratch {
  double* sum;     // [kSplits][C]
  int* kmax;       // [kSplits][C] ordered ints
  int* kmin;       // [kSplits][C]
  unsigned* amin;  // [kSplits][C] smallest nonzero |k| bits (0xFFFFFFFF: none)
  unsigned* words; // [0] max|v| bits, [1] max|K'| bits, [2] nonfinite flag
};

__host__ __device__ inline int64_t align256(int64_t x) { return (x + 255) / 256 * 256; }

__host__ __device__ inline Scratch scratch_at(uint8_t* base, int64_t C) {
  Scratch s;
  int64_t o = 0;
  s.sum = reinterpret_cast<double*>(base + o);
  o += align256((int64_t)kSplits * C * 8);
  s.kmax = reinterpret_cast<int*>(base + o);
  o += align256((int64_t)kSplits * C * 4);
  s.kmin = reinterpret_cast<int*>(base + o);
  o += align256((int64_t)kSplits * C * 4);
  s.amin = reinterpret_cast<unsigned*>(base + o);
  o += align256((int64_t)kSplits * C * 4);
  s.words = reinterpret_cast<unsigned*>(base + o);
  return s;
}

struct StatsParams {
  const uint8_t* k;
  const uint8_t* v;
  int64_t T, C;
  int64_t tokens_per_split;  // splits = gridDim.y
  Scratch sc;
};

__device__ __forceinline__ uint32_t max_s16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.s16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t min_s16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// bf16 value of an order-preserving int16 key (inverse of the key transform)
__device__ __forceinline__ float key_to_float(int key) {
  const uint32_t b = (uint32_t)(key < 0 ? (key ^ 0x7FFF) : key) & 0xFFFFu;
  return __uint_as_float(b << 16);
}

__global__ void __launch_bounds__(kStatsThreads) kv_stats_kernel(StatsParams p) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = (int64_t)blockIdx.x * kStatsCols + lane * 8;
  const bool active = c0 < p.C;
  const int split = blockIdx.y;
  const int64_t t_begin = (int64_t)split * p.tokens_per_split;
  const int64_t t_end = min(p.T, t_begin + p.tokens_per_split);

  // Per lane 8 columns = 4 words of two bf16.  The sums are doubles; max and min of
  // k are kept as order-preserving int16 keys (key = bits, with the magnitude bits
  // flipped for negative values) and the smallest nonzero |k| as |k| - 1 mod 2^15
  // (zero becomes 0x7FFF, above every nonzero magnitude), all two to a register.
  double sum[8];
  uint32_t kmx[4], kmn[4], amn[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) sum[i] = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    kmx[q] = 0x80008000u;
    kmn[q] = 0x7FFF7FFFu;
    amn[q] = 0x7FFF7FFFu;
  }
  unsigned vmax = 0;
  if (active) {
    constexpr int kRowStep = kStatsThreads / 32;
    for (int64_t t0 = t_begin + warp; t0 < t_end; t0 += kRowStep * kStatsUnroll) {
      uint4 kw[kStatsUnroll], vw[kStatsUnroll];
#pragma unroll
      for (int u = 0; u < kStatsUnroll; ++u) {
        const int64_t t = t0 + (int64_t)u * kRowStep;
        if (t < t_end) {
          kw[u] = ldg_nc_v4(p.k + (t * p.C + c0) * 2);
          vw[u] = ldg_nc_v4(p.v + (t * p.C + c0) * 2);
        }
      }
#pragma unroll
      for (int u = 0; u < kStatsUnroll; ++u) {
        if (t0 + (int64_t)u * kRowStep >= t_end) break;
        const uint32_t w[4] = {kw[u].x, kw[u].y, kw[u].z, kw[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t x = w[q];
          sum[2 * q] += (double)__uint_as_float(x << 16);
          sum[2 * q + 1] += (double)__uint_as_float(x & 0xFFFF0000u);
          const uint32_t key = x ^ (((x >> 15) & 0x00010001u) * 0x7FFFu);
          kmx[q] = max_s16x2(kmx[q], key);
          kmn[q] = min_s16x2(kmn[q], key);
          amn[q] = min_u16x2(amn[q], ((x & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x7FFF7FFFu);
        }
        vmax = __vmaxu2(vmax, vw[u].x & 0x7FFF7FFFu);
        vmax = __vmaxu2(vmax, vw[u].y & 0x7FFF7FFFu);
        vmax = __vmaxu2(vmax, vw[u].z & 0x7FFF7FFFu);
        vmax = __vmaxu2(vmax, vw[u].w & 0x7FFF7FFFu);
      }
    }
  }
  // back to floats and bit patterns per column; a key of +inf or above (+inf, +NaN)
  // or of -inf or below flags a non-finite k
  float kmax[8], kmin[8];
  unsigned amin[8];
  unsigned kbad = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int sh = 16 * (i & 1);
    const int hi = (int)(int16_t)(uint16_t)(kmx[i >> 1] >> sh);
    const int lo = (int)(int16_t)(uint16_t)(kmn[i >> 1] >> sh);
    const unsigned a16 = (amn[i >> 1] >> sh) & 0xFFFFu;
    kmax[i] = hi == -32768 ? -3.402823466e38f : key_to_float(hi);
    kmin[i] = lo == 32767 ? 3.402823466e38f : key_to_float(lo);
    amin[i] = a16 == 0x7FFFu ? 0xFFFFFFFFu : (a16 + 1u) << 16;
    if (hi >= 0x7F80 || lo <= (int)(int16_t)0x807F) kbad = 0x7F800000u;
  }
  vmax = max(vmax >> 16, vmax & 0xFFFFu) << 16;

  // cross-warp reduction in shared memory, warp-major
  __shared__ double s_sum[8][kStatsCols];
  __shared__ float s_max[8][kStatsCols];
  __shared__ float s_min[8][kStatsCols];
  __shared__ unsigned s_amin[8][kStatsCols];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    s_sum[warp][lane * 8 + i] = sum[i];
    s_max[warp][lane * 8 + i] = kmax[i];
    s_min[warp][lane * 8 + i] = kmin[i];
    s_amin[warp][lane * 8 + i] = amin[i];
  }
  __syncthreads();
  const int64_t col = (int64_t)blockIdx.x * kStatsCols + threadIdx.x;
  if (col < p.C) {
    double s = 0.0;
    float mx = -3.402823466e38f, mn = 3.402823466e38f;
    unsigned am = 0xFFFFFFFFu;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      s += s_sum[w][threadIdx.x];
      mx = fmaxf(mx, s_max[w][threadIdx.x]);
      mn = fminf(mn, s_min[w][threadIdx.x]);
      am = min(am, s_amin[w][threadIdx.x]);
    }
    const int64_t o = (int64_t)split * p.C + col;
    p.sc.sum[o] = s;
    p.sc.kmax[o] = float_to_ordered(mx);
    p.sc.kmin[o] = float_to_ordered(mn);
    p.sc.amin[o] = am;
  }
  // max|v| and the non-finite flag
  const unsigned vm = warp_max_u32(vmax);
  const unsigned kb = warp_max_u32(kbad);
  if (lane == 0) {
    if (vm) atomicMax(&p.sc.words[0], vm);
    if (vm >= 0x7F800000u || kb >= 0x7F800000u) atomicOr(&p.sc.words[2], 1u);
  }
}

// ------------------------------------------------------------- exact fallback

// Unsigned integer with 32-bit digits in uint64 slots (lazy carries).
constexpr int kLimbs = 10;

__device__ int limbs_bitlen(const unsigned long long* n) {
  for (int i = kLimbs - 1; i >= 0; --i)
    if (n[i]) return i * 32 + 32 - __clz((unsigned)n[i]);
  return 0;
}

// bit b of n (0 outside)
__device__ unsigned limbs_bit(const unsigned long long* n, int b) {
  if (b < 0 || b >= 32 * kLimbs) return 0;
  return (unsigned)(n[b >> 5] >> (b & 31)) & 1u;
}

// RN_f32(N * 2^-133 / T), N given by normalized limbs (digits < 2^32):
// take the top 64 bits of N (sticky for the rest), one 64-bit division by T
// (the integer part is the same as that of N / (T 2^sh)), then round.
__device__ float round_limbs_over_T(const unsigned long long* n, unsigned T, bool negative) {
  const int L = limbs_bitlen(n);
  if (L == 0) return 0.0f;
  const int sh = L - 64;  // N = top * 2^sh + low
  unsigned long long top = 0;
  for (int b = L - 1; b >= max(sh, 0); --b) top = (top << 1) | limbs_bit(n, b);
  if (sh < 0) top <<= -sh;
  bool sticky = false;
  for (int b = sh - 1; b >= 0 && !sticky; --b) sticky = limbs_bit(n, b);
  const unsigned long long q = top / T;
  sticky |= (top % T) != 0;
  const int lq = 64 - __clzll((long long)q);
  const int E = (lq - 1) + sh - 133;  // exponent of the leading bit
  const int lsb = max(E - 23, -149);
  // bits of q below the kept LSB: q has >= 33 significant bits, so a normal result
  // drops lq - 24 >= 9 of them; a subnormal one (E < -126 forces sh < 8 - lq)
  // drops -16 - sh, between 9 and 47.
  const int drop = lsb - (sh - 133);
  unsigned long long mant = q >> drop;
  const unsigned guard = (unsigned)(q >> (drop - 1)) & 1u;
  sticky |= (q & ((1ull << (drop - 1)) - 1ull)) != 0;
  if (guard && (sticky || (mant & 1ull))) ++mant;
  const float f = (float)ldexp((double)mant, lsb);
  return negative ? -f : f;
}

__device__ void limbs_normalize(unsigned long long* n) {
  for (int i = 0; i < kLimbs - 1; ++i) {
    n[i + 1] += n[i] >> 32;
    n[i] &= 0xFFFFFFFFull;
  }
}

// RN_f32(S / T) for an exactly known double S: one double division, then fix the
// only case where rounding twice can differ from rounding once — the double
// quotient q landing exactly halfway between two binary32 neighbours while S / T
// itself is not halfway.
__device__ float mean_from_exact_double(double S, unsigned T) {
  const double q = S / (double)T;
  const float f = (float)q;
  const double fd = (double)f;
  if (q != fd) {
    const float nb = q > fd ? nextafterf(f, 3.402823466e38f) : nextafterf(f, -3.402823466e38f);
    if (q == 0.5 * (fd + (double)nb)) {
      const double r = fma(-q, (double)T, S);  // exact sign of S/T - q
      if (r != 0.0) return r > 0.0 ? fmaxf(f, nb) : fminf(f, nb);
    }
  }
  return f;
}

struct MuParams {
  const uint8_t* k;
  int64_t T, C;
  int nsplits;
  Scratch sc;
  float* mu;   // slot's mu [C]
  int log2T_ceil;
};

// kMuCols columns per CTA: warp w folds splits w, w + 8, ... of every column (lane
// = column), warp 0 combines the 8 partial results.  When a column passes the
// range test every partial sum is an exact double, so the order of the additions
// does not matter.
__global__ void __launch_bounds__(kMuThreads) kv_mu_kernel(MuParams p) {
  pdl_trigger();
  pdl_wait();
  if (p.sc.words[2]) return;  // non-finite input: the slot stays unchanged
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kMuThreads / 32;
  const int64_t c = (int64_t)blockIdx.x * kMuCols + lane;
  __shared__ double r_sum[kWarps][kMuCols];
  __shared__ float r_max[kWarps][kMuCols];
  __shared__ float r_min[kWarps][kMuCols];
  __shared__ unsigned r_amin[kWarps][kMuCols];
  __shared__ int n_inexact;
  __shared__ int inexact_cols[kMuCols];
  __shared__ float inexact_mu[kMuCols];
  __shared__ unsigned long long limbs[2][kLimbs];
  if (threadIdx.x == 0) n_inexact = 0;
  {
    double S = 0.0;
    float mx = -3.402823466e38f, mn = 3.402823466e38f;
    unsigned am = 0xFFFFFFFFu;
    if (c < p.C) {
#pragma unroll 4
      for (int sp = warp; sp < p.nsplits; sp += kWarps) {
        const int64_t o = (int64_t)sp * p.C + c;
        S += p.sc.sum[o];
        mx = fmaxf(mx, ordered_to_float(p.sc.kmax[o]));
        mn = fminf(mn, ordered_to_float(p.sc.kmin[o]));
        am = min(am, p.sc.amin[o]);
      }
    }
    r_sum[warp][lane] = S;
    r_max[warp][lane] = mx;
    r_min[warp][lane] = mn;
    r_amin[warp][lane] = am;
  }
  __syncthreads();
  double S = 0.0;
  float kmax = -3.402823466e38f, kmin = 3.402823466e38f;
  unsigned amin = 0xFFFFFFFFu;
  bool exact = true;
  if (warp == 0 && c < p.C) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      S += r_sum[w][lane];
      kmax = fmaxf(kmax, r_max[w][lane]);
      kmin = fminf(kmin, r_min[w][lane]);
      amin = min(amin, r_amin[w][lane]);
    }
    if (amin != 0xFFFFFFFFu) {
      const float amax = fmaxf(fabsf(kmax), fabsf(kmin));
      const int e_max = max((int)((__float_as_uint(amax) >> 23) & 0xFF), 1);
      const int e_min = max((int)((amin >> 23) & 0xFF), 1);
      exact = (e_max - e_min) <= 45 - p.log2T_ceil;
    }
    if (!exact) inexact_cols[atomicAdd(&n_inexact, 1)] = lane;
  }
  __syncthreads();
  // exact integer-limb sums for the (rare) columns outside the double's range
  const int n_in = n_inexact;
  for (int i = 0; i < n_in; ++i) {
    const int64_t cc = (int64_t)blockIdx.x * kMuCols + inexact_cols[i];
    if (threadIdx.x < 2 * kLimbs) limbs[threadIdx.x / kLimbs][threadIdx.x % kLimbs] = 0;
    __syncthreads();
    for (int64_t t = threadIdx.x; t < p.T; t += kMuThreads) {
      const unsigned b = *reinterpret_cast<const unsigned short*>(p.k + (t * p.C + cc) * 2);
      const unsigned e = (b >> 7) & 0xFFu, m = b & 0x7Fu;
      if (e == 0 && m == 0) continue;
      const unsigned long long mant = e ? (128u + m) : m;  // value = mant * 2^(pos - 133)
      const int pos = e ? (int)e - 1 : 0;
      atomicAdd(&limbs[b >> 15][pos >> 5], mant << (pos & 31));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      unsigned long long* P = limbs[0];
      unsigned long long* N = limbs[1];
      limbs_normalize(P);
      limbs_normalize(N);
      int cmp = 0;
      for (int d = kLimbs - 1; d >= 0 && cmp == 0; --d)
        cmp = P[d] > N[d] ? 1 : (P[d] < N[d] ? -1 : 0);
      unsigned long long mag[kLimbs];
      const unsigned long long* big = cmp >= 0 ? P : N;
      const unsigned long long* small = cmp >= 0 ? N : P;
      long long borrow = 0;
      for (int d = 0; d < kLimbs; ++d) {
        long long t = (long long)big[d] - (long long)small[d] - borrow;
        borrow = t < 0;
        mag[d] = (unsigned long long)(t + (borrow ? (1ll << 32) : 0));
      }
      inexact_mu[i] = cmp == 0 ? 0.0f : round_limbs_over_T(mag, (unsigned)p.T, cmp < 0);
    }
    __syncthreads();
  }
  if (warp != 0 || c >= p.C) return;
  float mu;
  if (!exact) {
    mu = 0.0f;
    for (int i = 0; i < n_in; ++i)
      if (inexact_cols[i] == lane) mu = inexact_mu[i];
  } else {
    mu = (amin == 0xFFFFFFFFu) ? 0.0f : mean_from_exact_double(S, (unsigned)p.T);
  }
  p.mu[c] = mu;
  // max |RN(k - mu)| over the column is reached at its max or its min (RN is monotone)
  const float a = fmaxf(fabsf(kmax - mu), fabsf(kmin - mu));
  atomicMax(&p.sc.words[1], __float_as_uint(a));
}

struct EncParams {
  const uint8_t* k;
  const uint8_t* v;
  int64_t nblocks;    // T * C / 16
  FastDiv cblocks;    // C / 16
  const float* mu;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint8_t* k_scales;
  uint8_t* v_scales;
  float* gscale;      // slot's (g_K, g_V)
  int32_t* slot_tokens;  // slot's recorded token count
  int32_t tokens;
  const unsigned* words;
  unsigned* status;
};

__device__ __forceinline__ void encode_block16(const float (&v)[16], float g, float d6, float r6,
                                               uint8_t* codes, uint8_t* scale) {
  float v0[8], v1[8];
  float amax_b = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax_b = fmaxf(amax_b, fabsf(v[k]));
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v0[k] = v[k];
    v1[k] = v[8 + k];
  }
  const uint32_t s = block_scale_fast(amax_b, d6, r6);
  const BlockEncoder enc(e4m3_to_float(s) * g);
  uint2 out;
  // scalar bracket products here: the paired form costs this kernel a resident CTA
  // per SM (66 registers), which measured slower
  out.x = enc.encode8s<false>(v0);
  out.y = enc.encode8s<false>(v1);
  stg_v2(codes, out);
  *scale = (uint8_t)s;
}

__global__ void __launch_bounds__(kEncThreads) kv_encode_kernel(EncParams p) {
  pdl_trigger();
  pdl_wait();
  if (p.words[2]) {  // a NaN or Inf in K or V: report it, leave the slot unchanged
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(p.status, kStatusNonfinite);
    return;
  }
  const float gk = __uint_as_float(p.words[1]) / 2688.0f;
  const float gv = __uint_as_float(p.words[0]) / 2688.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.gscale[0] = gk;
    p.gscale[1] = gv;
    *p.slot_tokens = p.tokens;
  }
  const float d6k = 6.0f * gk, d6v = 6.0f * gv;
  const float r6k = 1.0f / d6k, r6v = 1.0f / d6v;
  const int64_t stride = (int64_t)gridDim.x * kEncThreads;
  for (int64_t b = (int64_t)blockIdx.x * kEncThreads + threadIdx.x; b < p.nblocks; b += stride) {
    const uint32_t row = p.cblocks.div((uint32_t)b);
    const int64_t c = ((int64_t)b - (int64_t)row * p.cblocks.d) * 16;
    float kv[16], vv[16];
    {
      const uint4 a = ldg_nc_v4_l1(p.k + b * 32), bb = ldg_nc_v4_l1(p.k + b * 32 + 16);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
      const float4* m4 = reinterpret_cast<const float4*>(p.mu + c);
      float mu[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 m = m4[q];
        mu[4 * q] = m.x;
        mu[4 * q + 1] = m.y;
        mu[4 * q + 2] = m.z;
        mu[4 * q + 3] = m.w;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        kv[2 * q] = bf16_lo(w[q]) - mu[2 * q];
        kv[2 * q + 1] = bf16_hi(w[q]) - mu[2 * q + 1];
      }
    }
    {
      const uint4 a = ldg_nc_v4_l1(p.v + b * 32), bb = ldg_nc_v4_l1(p.v + b * 32 + 16);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        vv[2 * q] = bf16_lo(w[q]);
        vv[2 * q + 1] = bf16_hi(w[q]);
      }
    }
    encode_block16(kv, gk, d6k, r6k, p.k_codes + b * 8, p.k_scales + b);
    encode_block16(vv, gv, d6v, r6v, p.v_codes + b * 8, p.v_scales + b);
  }
}

struct WindowParams {
  const uint8_t* base;
  int64_t off_k_codes, off_v_codes, off_k_scales, off_v_scales, off_mu, off_gscale, off_tokens;
  int64_t slot_codes_bytes, slot_scales_bytes, C;
  FastDiv cblocks;           // C / 16
  int32_t n_slots;
  int32_t slots[kMaxWindowSlots];
  int32_t tokens[kMaxWindowSlots];
  int64_t hb_end[kMaxWindowSlots];  // cumulative half-blocks (8 values) through list entry i
  uint8_t* k_out;
  uint8_t* v_out;
  unsigned* status;
};

// One flat sweep over the output (the listed slots' tokens one after the other),
// two threads per 16-value block of K and of V (8 values each): half-block hb of
// the output is written at byte 16 hb of k_out / v_out.  A thread tracks the list
// entry its index falls in and moves on as its index advances.
__global__ void __launch_bounds__(kEncThreads) kv_window_kernel(WindowParams p) {
  pdl_trigger();
  pdl_wait();
  const int64_t total = p.hb_end[p.n_slots - 1];
  const int64_t stride = (int64_t)gridDim.x * kEncThreads;
  int i = -1;
  int64_t begin = 0, end = 0, slot = 0;
  bool ok = false;
  float gk = 0.0f, gv = 0.0f;
  for (int64_t hb = (int64_t)blockIdx.x * kEncThreads + threadIdx.x; hb < total; hb += stride) {
    while (hb >= end) {  // next list entry (a stride may skip short ones)
      ++i;
      begin = end;
      end = p.hb_end[i];
      slot = p.slots[i];
      ok = reinterpret_cast<const int32_t*>(p.base + p.off_tokens)[slot] == p.tokens[i];
      if (!ok && hb == begin) set_status(p.status, kStatusShape);
      const float* g = reinterpret_cast<const float*>(p.base + p.off_gscale) + 2 * slot;
      gk = g[0];
      gv = g[1];
    }
    if (!ok) continue;
    const int64_t lh = hb - begin;  // half-block within the slot
    const int64_t b = lh >> 1;
    const int half = (int)(lh & 1);
    const uint32_t row = p.cblocks.div((uint32_t)b);
    const int64_t c = (b - (int64_t)row * p.cblocks.d) * 16 + half * 8;
    const int64_t cofs = slot * p.slot_codes_bytes + lh * 4, sofs = slot * p.slot_scales_bytes + b;
    const uint32_t kc = *reinterpret_cast<const uint32_t*>(p.base + p.off_k_codes + cofs);
    const uint32_t vc = *reinterpret_cast<const uint32_t*>(p.base + p.off_v_codes + cofs);
    const uint32_t ks2 = e4m3_to_f16x2_bcast(p.base[p.off_k_scales + sofs]);
    const uint32_t vs2 = e4m3_to_f16x2_bcast(p.base[p.off_v_scales + sofs]);
    const float4* m4 = reinterpret_cast<const float4*>(p.base + p.off_mu + (slot * p.C + c) * 4);
    const float4 m0 = m4[0], m1 = m4[1];
    const float mu[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    uint32_t kh[4], vh[4];
    e2m1x8_times_scale(kc, ks2, kh);
    e2m1x8_times_scale(vc, vs2, vh);
    float ko[8], vo[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f16x2_to_f32x2(kh[q], ko[2 * q], ko[2 * q + 1]);  // e2m1 * s, exact
      f16x2_to_f32x2(vh[q], vo[2 * q], vo[2 * q + 1]);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      ko[q] = ko[q] * gk + mu[q];  // no fusion: -fmad=false
      vo[q] = vo[q] * gv;
    }
    stg_v4(p.k_out + hb * 16, make_uint4(pack_bf16x2(ko[0], ko[1]), pack_bf16x2(ko[2], ko[3]),
                                         pack_bf16x2(ko[4], ko[5]), pack_bf16x2(ko[6], ko[7])));
    stg_v4(p.v_out + hb * 16, make_uint4(pack_bf16x2(vo[0], vo[1]), pack_bf16x2(vo[2], vo[3]),
                                         pack_bf16x2(vo[4], vo[5]), pack_bf16x2(vo[6], vo[7])));
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Stats -> mu -> encode for one append, statistics in `sc` (words already zeroed).
// The token splits of the stats pass fill one wave of resident CTAs (at most
// kSplits, the size the scratch is laid out for).
cudaError_t launch_append_kernels(const KVLayout& L, const void* k, const void* v, int64_t T, int32_t slot,
                                  const Scratch& sc, unsigned* status, cudaStream_t s) {
  const int64_t C = (int64_t)L.heads * L.head_dim;
  static std::atomic<int> resident[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (resident[dev].load(std::memory_order_relaxed) == 0) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kv_stats_kernel, kStatsThreads, 0);
    if (e != cudaSuccess) return e;
    resident[dev].store(max(1, per_sm) * sm_count(), std::memory_order_relaxed);
  }
  const int64_t colblocks = (C + kStatsCols - 1) / kStatsCols;
  const int64_t resident_now = resident[dev].load(std::memory_order_relaxed);
  const int nsplits = (int)max((int64_t)1, min((int64_t)kSplits, resident_now / colblocks));

  StatsParams sp;
  sp.k = (const uint8_t*)k;
  sp.v = (const uint8_t*)v;
  sp.T = T;
  sp.C = C;
  sp.tokens_per_split = (T + nsplits - 1) / nsplits;
  sp.sc = sc;
  dim3 sgrid((unsigned)colblocks, (unsigned)nsplits);
  launch_pdl(kv_stats_kernel, sgrid, kStatsThreads, 0, s, sp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  MuParams mp;
  mp.k = (const uint8_t*)k;
  mp.T = T;
  mp.C = C;
  mp.nsplits = nsplits;
  mp.sc = sc;
  mp.mu = reinterpret_cast<float*>(L.base + L.off_mu) + (int64_t)slot * C;
  int lg = 0;
  while ((1ll << lg) < T) ++lg;
  mp.log2T_ceil = lg;
  launch_pdl(kv_mu_kernel, (unsigned)((C + kMuCols - 1) / kMuCols), kMuThreads, 0, s, mp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  EncParams ep;
  ep.k = (const uint8_t*)k;
  ep.v = (const uint8_t*)v;
  ep.nblocks = T * C / 16;
  ep.cblocks = FastDiv((uint32_t)(C / 16));
  ep.mu = mp.mu;
  ep.k_codes = L.base + L.off_k_codes + (int64_t)slot * L.slot_codes_bytes;
  ep.v_codes = L.base + L.off_v_codes + (int64_t)slot * L.slot_codes_bytes;
  ep.k_scales = L.base + L.off_k_scales + (int64_t)slot * L.slot_scales_bytes;
  ep.v_scales = L.base + L.off_v_scales + (int64_t)slot * L.slot_scales_bytes;
  ep.gscale = reinterpret_cast<float*>(L.base + L.off_gscale) + 2 * (int64_t)slot;
  ep.slot_tokens = reinterpret_cast<int32_t*>(L.base + L.off_tokens) + slot;
  ep.tokens = (int32_t)T;
  ep.words = sc.words;
  ep.status = status;
  launch_pdl(kv_encode_kernel, wave_grid<kv_encode_kernel>(kEncThreads, ep.nblocks), kEncThreads, 0, s, ep);
  return cudaGetLastError();
}

}  // namespace

int64_t kv_scratch_bytes(int32_t heads, int32_t head_dim, int64_t chunk_tokens) {
  (void)chunk_tokens;
  const int64_t C = (int64_t)heads * head_dim;
  return align256((int64_t)kSplits * C * 8) + 3 * align256((int64_t)kSplits * C * 4) + 256;
}

cudaError_t launch_kv_append(const KVLayout& L, const void* k, const void* v, int64_t tokens, int32_t slot,
                             unsigned* status, cudaStream_t s) {
  const int64_t C = (int64_t)L.heads * L.head_dim;
  Scratch sc = scratch_at(L.base + L.off_scratch, C);
  cudaError_t e = launch_zero_words(sc.words, 3, s);
  if (e != cudaSuccess) return e;

  return launch_append_kernels(L, k, v, tokens, slot, sc, status, s);
}

cudaError_t launch_kv_window(const KVLayout& L, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                             void* k_out, void* v_out, unsigned* status, cudaStream_t s) {
  WindowParams p;
  p.base = L.base;
  p.off_k_codes = L.off_k_codes;
  p.off_v_codes = L.off_v_codes;
  p.off_k_scales = L.off_k_scales;
  p.off_v_scales = L.off_v_scales;
  p.off_mu = L.off_mu;
  p.off_gscale = L.off_gscale;
  p.off_tokens = L.off_tokens;
  p.slot_codes_bytes = L.slot_codes_bytes;
  p.slot_scales_bytes = L.slot_scales_bytes;
  p.C = (int64_t)L.heads * L.head_dim;
  p.cblocks = FastDiv((uint32_t)(p.C / 16));
  int64_t acc = 0;
  p.n_slots = n_slots;
  for (int i = 0; i < n_slots; ++i) {
    p.slots[i] = slots[i];
    p.tokens[i] = tokens[i];
    acc += (int64_t)tokens[i] * p.C / 8;
    p.hb_end[i] = acc;
  }
  p.k_out = static_cast<uint8_t*>(k_out);
  p.v_out = static_cast<uint8_t*>(v_out);
  p.status = status;
  const int grid = wave_grid<kv_window_kernel>(kEncThreads, acc);
  launch_pdl(kv_window_kernel, grid, kEncThreads, 0, s, p);
  return cudaGetLastError();
}

// ------------------------------------------------- append without caller scratch
// Statistics scratch of kv_quant_append_noalloc: one static array per device that
// loads the library, sized for at most kNoAllocMaxColumns = heads * head_dim
// columns (64 token splits x 20 bytes per column, plus three words): 5.0 MiB.
// Host code must not use this name as an address; it asks the runtime for the
// device address of the current device's copy once (kv_noalloc_scratch).
static __device__ __align__(256) uint8_t g_kv_noalloc_scratch[
    (kSplits * kNoAllocMaxColumns * 8) + 3 * (kSplits * kNoAllocMaxColumns * 4) + 256];

static_assert(kSplits * kNoAllocMaxColumns * 8 % 256 == 0 && kSplits * kNoAllocMaxColumns * 4 % 256 == 0,
              "scratch_at's 256-byte alignment must leave the static array's layout unpadded");

namespace {
std::mutex g_noalloc_mu;
uint8_t* g_noalloc_ptr[64];
}  // namespace

// Device address of this device's static scratch array (looked up once per device,
// with that device current).
static cudaError_t kv_noalloc_scratch(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kv_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

cudaError_t launch_kv_append_noalloc(const KVLayout& L, const void* k, const void* v, int64_t tokens,
                                     int32_t slot, unsigned* status, cudaStream_t s) {
  const int64_t C = (int64_t)L.heads * L.head_dim;
  if (C > kNoAllocMaxColumns) return cudaErrorInvalidValue;
  uint8_t* scratch = nullptr;
  cudaError_t e = kv_noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  Scratch sc = scratch_at(scratch, C);
  // the words accumulate with atomics: they must start at zero on every call; the
  // statistics of every split in use are fully rewritten by kv_stats_kernel
  if ((e = launch_zero_words(sc.words, 3, s)) != cudaSuccess) return e;

  return launch_append_kernels(L, k, v, tokens, slot, sc, status, s);
}

}  // namespace nvfp4
