// common.cuh — device helpers shared by the libnvfp4 kernels (sm_100a).
//
// Number format, as fixed by the library (techwalker.com, "NVIDIA研究团队打造全球首个FP4视频
// 生成系统，速度提升两倍还省一半内存", §一: 4-bit E2M1 values, one FP8 scale per 16 values,
// one FP32 scale for the whole tensor):
//   g  = RN(amax / 2688)                       tensor scale (2688 = 6 * 448)
//   s  = E4M3_RNE_sat(RN(amax_b / RN(6 g)))    block scale, one byte per 16 values
//   D  = RN(value(s) * g)
//   code = sign(x) | E2M1 round-to-nearest-even of the exact quotient |x| / D
// All arithmetic here is IEEE binary32 round-to-nearest-even; the library is
// compiled with -fmad=false so no product/sum pair is silently fused, and every
// intended fused multiply-add is written as fmaf().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

enum : unsigned { kStatusOk = 0, kStatusShape = 2, kStatusNonfinite = 4, kStatusTimeout = 5 };

// The first data error wins; later ones leave the word unchanged (sticky).
__device__ __forceinline__ void set_status(unsigned* status, unsigned code) {
  atomicCAS(status, 0u, code);
}

// ---------------------------------------------------------------- loads/stores
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Read-only 16-byte load that may allocate in L1: for access patterns where one
// warp instruction uses half of each 32-byte sector and the next uses the rest.
__device__ __forceinline__ uint4 ldg_nc_v4_l1(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void stg_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void stg_v2(void* p, uint2 v) {
  asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// ---------------------------------------------------------------- bf16 / fp32
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// two floats -> packed bf16x2 (RNE); `lo` lands in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- E4M3
// RNE with saturation to 448 of a finite s >= 0 (hardware conversion).
__device__ __forceinline__ uint32_t e4m3_from_float(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return (uint32_t)(r & 0xFFu);
}

// Value of an E4M3 byte (never NaN here), through the exact E4M3 -> f16 -> f32
// hardware conversions.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  uint32_t h2;
  float f;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)b));
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"((uint16_t)(h2 & 0xFFFFu)));
  return f;
}

// Hardware reciprocal approximation (at most 1 ulp from 1/x for normal x).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Programmatic dependent launch: every kernel of the library is launched so that
// the next one may start before it ends.  pdl_trigger lets the grid launched after
// this one on the stream begin (its CTAs then wait in pdl_wait); pdl_wait blocks
// until every grid before this one on the stream has completed and its memory is
// visible, so it goes before the first read of anything a previous kernel wrote.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- grid barrier
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

constexpr unsigned long long kGridBarrierLimitNs = 2000000000ull;

// Barrier of a whole grid whose CTAs are all resident at once (one wave, sized by
// the occupancy query, launched after every earlier grid on the stream has
// started).  *ctr is zero before the launch; each CTA adds one and waits for
// `expected` arrivals (every CTA of the grid).  The wait is bounded: false after limit_ns, and the caller
// records a timeout instead of hanging.  Memory written by any CTA before the
// barrier is visible to every CTA after it (release/acquire at GPU scope).
__device__ __forceinline__ bool grid_barrier_n(unsigned* ctr, unsigned expected, unsigned long long limit_ns) {
  __shared__ int barrier_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    int ok = 1;
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_gpu(ctr) < expected) {
      if (globaltimer_ns() - t0 > limit_ns) {
        ok = 0;
        break;
      }
      __nanosleep(100);
    }
    barrier_ok = ok;
  }
  __syncthreads();
  return barrier_ok != 0;
}

// ---------------------------------------------------------------- E2M1
// Exact E2M1 magnitude index of |x| / D by comparing |x| with each midpoint
// m * D (m = 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5).  fmaf gives the correctly
// rounded |x| - m D, whose sign is exact whenever D >= 2^-100 (the difference is
// then either 0 or far above the binary32 underflow threshold).  A tie counts
// toward the even neighbour: "> 0" where the lower index is even, ">= 0" where
// the upper one is.
__device__ __forceinline__ uint32_t e2m1_index_exact(float ax, float D) {
  uint32_t i = 0;
  i += fmaf(-0.25f, D, ax) > 0.0f;
  i += fmaf(-0.75f, D, ax) >= 0.0f;
  i += fmaf(-1.25f, D, ax) > 0.0f;
  i += fmaf(-1.75f, D, ax) >= 0.0f;
  i += fmaf(-2.5f, D, ax) > 0.0f;
  i += fmaf(-3.5f, D, ax) >= 0.0f;
  i += fmaf(-5.0f, D, ax) > 0.0f;
  return i;
}

// Same decision in double for tiny D (every m * D is exact in double).
static __device__ __noinline__ uint32_t e2m1_index_exact_f64(float ax, float D) {
  const double a = ax, d = D;
  uint32_t i = 0;
  i += a > 0.25 * d;
  i += a >= 0.75 * d;
  i += a > 1.25 * d;
  i += a >= 1.75 * d;
  i += a > 2.5 * d;
  i += a >= 3.5 * d;
  i += a > 5.0 * d;
  return i;
}


// Block encoder: D = RN(s * g) and rD ~ 1 / D (hardware reciprocal, <= 1 ulp) are
// computed once per block, and from rD two brackets rDlo < 1 / D < rDhi (rD scaled
// by 1 -+ 2^-20, whose RN errors stay below 2^-23 + 2^-24).  For an element x the
// exact quotient x / D then lies strictly between RN(x rDlo) and RN(x rDhi), and
// E2M1 round-to-nearest-even (the hardware cvt, sign in bit 3 also for values
// that round to zero) is monotonic: where both brackets give the same code it is
// the code of the exact quotient.  Elements whose brackets differ (x / D within
// ~2^-20 of an E2M1 midpoint, ties included) take the exact comparison path.
// Two-lane FP32 arithmetic (the .f32x2 forms of sm_100): each lane rounds to nearest
// even exactly like the scalar operation, so a pair of results is bit-identical to two
// scalar operations, at one instruction instead of two.  A paired multiply whose result
// feeds a paired add may still be contracted into one fused multiply-add by the
// assembler (seen on sm_100a: a single rounding where two were written), so wherever the
// intermediate rounding is part of the defined result, write the two steps with
// __fmul_rn and __fadd_rn instead.
__device__ __forceinline__ void mul2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

struct BlockEncoder {
  float D, rD;
  bool tiny;  // D < 2^-100 or D > 2^125 (1/D near the flushed range): exact path for the whole block

  float rDlo, rDhi;

  __device__ __forceinline__ BlockEncoder(float D_) : D(D_) {
    rD = (D > 0.0f) ? rcp_approx(D) : 0.0f;
    rDlo = rD * 0.99999904632568359375f;  // 1 - 2^-20
    rDhi = rD * 1.00000095367431640625f;  // 1 + 2^-20
    tiny = D < 7.8886090522101181e-31f || D > 4.2535295865117308e37f;  // 2^-100, 2^125
  }

  __device__ __forceinline__ uint32_t index_slow(float ax) const {
    return tiny ? e2m1_index_exact_f64(ax, D) : e2m1_index_exact(ax, D);
  }

  // 8 signed values -> 8 E2M1 codes packed into 32 bits (element k in bits 4k..4k+3).
  // kPaired: bracket products as two-lane FP32 multiplies (fewer instructions, two
  // more registers); the results are the same either way.
  template <bool kPaired = true>
  __device__ __forceinline__ uint32_t encode8s(const float (&v)[8]) const;
};

// Per-block scale: s = E4M3_RNE_sat(RN(amax_b / d6)) with d6 = RN(6 g); d6 == 0 -> 0.
__device__ __forceinline__ uint32_t block_scale(float amax_b, float d6) {
  if (!(d6 > 0.0f)) return 0u;
  return e4m3_from_float(amax_b / d6);
}

// The same scale from the product t = RN(amax_b * r6), r6 = RN(1 / d6): t is within
// 1.5 ulp of RN(amax_b / d6), so both round to the same E4M3 value unless an E4M3
// rounding boundary lies within a few ulp of t.  In the normal range (t >= 2^-6)
// those boundaries have binary32 fraction bits 19..0 = 0x80000 and are never a
// power of two; t in the subnormal range, non-finite, or within 4 ulp of a
// boundary takes the division.
__device__ __forceinline__ uint32_t block_scale_fast(float amax_b, float d6, float r6) {
  if (!(d6 > 0.0f)) return 0u;
  const float t = amax_b * r6;
  const uint32_t u = __float_as_uint(t);
  if (!(t >= 0.015625f && t < 1.0e30f) || ((u + 0x80004u) & 0xFFFFFu) <= 8u) return e4m3_from_float(amax_b / d6);
  return e4m3_from_float(t);
}

// Sign bits of 8 floats -> bit 3 of each nibble (so -0 encodes as 0x8).
__device__ __forceinline__ uint32_t f32_signs8(const float (&v)[8]) {
  uint32_t r = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) r |= (__float_as_uint(v[k]) >> 31) << (4 * k + 3);
  return r;
}

// 8 values -> 8 codes, element k in bits 4k..4k+3: four paired conversions whose
// bytes are packed by one vector move.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float (&q)[8]) {
  uint32_t word;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(word)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return word;
}

template <bool kPaired>
__device__ __forceinline__ uint32_t BlockEncoder::encode8s(const float (&v)[8]) const {
  if (!(D > 0.0f)) return f32_signs8(v);  // every magnitude index is 0
  float ql[8], qh[8];
  if constexpr (kPaired) {
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      mul2(ql[k], ql[k + 1], v[k], v[k + 1], rDlo, rDlo);
      mul2(qh[k], qh[k + 1], v[k], v[k + 1], rDhi, rDhi);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      ql[k] = v[k] * rDlo;
      qh[k] = v[k] * rDhi;
    }
  }
  uint32_t word = pack_e2m1x8(ql);
  const uint32_t wh = pack_e2m1x8(qh);
  if (tiny || word != wh) {
    const uint32_t diff = tiny ? 0xFFFFFFFFu : (word ^ wh);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if ((diff >> (4 * k)) & 0xFu) {
        const uint32_t c = index_slow(fabsf(v[k])) | ((__float_as_uint(v[k]) >> 31) << 3);
        word = (word & ~(0xFu << (4 * k))) | (c << (4 * k));
      }
    }
  }
  return word;
}

// E4M3 byte -> the same value in both halves of an f16x2 (exact conversion).
__device__ __forceinline__ uint32_t e4m3_to_f16x2_bcast(uint32_t b) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(b | (b << 8))));
  return h2;
}

// Eight E2M1 codes (one 32-bit word, element k in bits 4k..4k+3) times a block
// scale given as f16x2: four f16x2 products, element 2i in the low half of p[i].
// The hardware E2M1 -> f16 conversion is exact, and so is the f16 product: the
// magnitudes e2m1 * s lie in [2^-10, 6 * 448] with at most 6 significant bits.
__device__ __forceinline__ void e2m1x8_times_scale(uint32_t w, uint32_t s2, uint32_t (&p)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 h0, h1, h2, h3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 h0, b0;\n\tcvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 h2, b2;\n\tcvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
      "mul.rn.f16x2 %0, h0, %5;\n\tmul.rn.f16x2 %1, h1, %5;\n\t"
      "mul.rn.f16x2 %2, h2, %5;\n\tmul.rn.f16x2 %3, h3, %5;\n\t}"
      : "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3])
      : "r"(w), "r"(s2));
}

// f16x2 -> its two halves as floats (exact).
__device__ __forceinline__ void f16x2_to_f32x2(uint32_t h, float& lo, float& hi) {
  asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h));
}

// Offset of block scale (r, j) in the tensor-core (MMA) scale layout.
__device__ __forceinline__ int64_t sf_mma_offset(int64_t r, int64_t j, int64_t groups) {
  return ((r >> 7) * groups + (j >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (j & 3);
}

// Float <-> order-preserving signed int (for atomicMin/atomicMax on floats).
__device__ __forceinline__ int float_to_ordered(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ordered_to_float(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF);
}

// Warp reductions
__device__ __forceinline__ unsigned warp_max_u32(unsigned v) { return __reduce_max_sync(0xFFFFFFFFu, v); }

// Fast unsigned division of 32-bit values by a runtime constant d >= 1
// (round-up multiplier method, Granlund & Montgomery 1994):
//   l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
//   n / d = (t + ((n - t) >> 1)) >> (l - 1) with t = umulhi(n, m)   (d > 1).
struct FastDiv {
  uint32_t d, m, l;
  __host__ FastDiv() : d(1), m(1), l(0) {}
  __host__ explicit FastDiv(uint32_t d_) : d(d_), m(1), l(0) {
    while ((1ull << l) < d) ++l;
    m = (uint32_t)((((1ull << 32) * ((1ull << l) - d)) / d) + 1);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    if (d == 1) return n;
    const uint32_t t = __umulhi(n, m);
    return (t + ((n - t) >> 1)) >> (l - 1);
  }
};

}  // namespace nvfp4
