/*
 * nvfp4_oracle.c — ORACLE: plain, slow, obviously correct CPU statement of the
 * NVFP4 hot path.  This is TEST INFRASTRUCTURE.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load it.  It shares no code, table or
 * header with the CUDA library, and the CUDA library never calls it.
 *
 * Built with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math (no FMA
 * contraction, no flush-to-zero; float arithmetic is IEEE binary32 with
 * round-to-nearest-even, written RN below).
 *
 * Sources (web pages about LongLive-2.0):
 *   [TW §一] techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存",
 *            §一: every 16 values share one FP8 scale, the whole tensor shares one FP32
 *            scale; values are E2M1 (non-uniform spacing).
 *   [TW §四] same page, §四: K has its mean subtracted before NVFP4 storage; several
 *            cache chunks are dequantized together.
 * Readings fixed where the pages are silent (the E4M3 flavour of "FP8", the scale
 * formulas, the rounding rules, the per-(head,dim) mean over the chunk) are stated
 * at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_NONFINITE 4
#define ORACLE_ERR_ARG 1

/* ----------------------------------------------------------- scalar formats */

/* E2M1 magnitudes: 2 exponent bits (bias 1), 1 mantissa bit; code 0..7. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Value of a 4-bit E2M1 code; bit 3 is the sign.  [TW §一] */
double oracle_e2m1_value(uint8_t code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* E2M1 magnitude index of the EXACT real quotient ax / D (ax >= 0, D > 0):
 * the nearest magnitude, ties to the even index, saturating at 6.
 * Each midpoint times D has at most 3 + 24 significant bits, so the products
 * below are exact in double and every comparison is exact. */
int oracle_e2m1_index_exact(float ax, float D) {
  if (!(D > 0.0f)) return 0;
  for (int i = 0; i < 7; ++i) {
    double t = 0.5 * (E2M1_MAG[i] + E2M1_MAG[i + 1]) * (double)D;
    if ((double)ax < t) return i;
    if ((double)ax == t) return (i % 2 == 0) ? i : i + 1;
  }
  return 7;
}

/* Value of an E4M3FN byte: bias 7, exponent field 0 = subnormal (m/8 * 2^-6),
 * S.1111.111 = NaN, no infinities. */
double oracle_e4m3_value(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return s ? -v : v;
}

/* E4M3 round-to-nearest-even with saturation to the largest finite value (448),
 * for a finite s >= 0: brute force over the 127 non-negative finite codes; on a
 * tie the code with the even mantissa (even code) wins. */
uint8_t oracle_e4m3_encode(float s) {
  if (!(s >= 0.0f)) return 0;
  if (s >= 448.0f) return 0x7E;
  uint8_t best = 0;
  double bestd = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(oracle_e4m3_value((uint8_t)c) - (double)s);
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      bestd = d;
      best = (uint8_t)c;
    }
  }
  return best;
}

float oracle_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* bf16 round-to-nearest-even of a finite float (carry into the exponent is the
 * correct behaviour at a binade edge). */
uint16_t oracle_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static float load_elem(const void* x, int xt, int64_t idx) {
  if (xt == 0) return oracle_bf16_to_f32(((const uint16_t*)x)[idx]);
  return ((const float*)x)[idx];
}

/* ----------------------------------------------------------- quantize */

/* NVFP4 quantization of x [rows, cols] (xt: 0 = bf16 bits, 1 = float),
 * leading dimension ldx elements.  Outputs (row-major, canonical):
 *   codes  [rows, cols/2]  element 2i in the low nibble of byte i
 *   scales [rows, cols/16] E4M3 bytes
 *   *g_out tensor scale, *amax_out = max|x|.
 * gscale_in: NULL -> g = RN(amax / 2688); else g = *gscale_in (host value).
 * Steps:  [TW §一]
 *   1. any NaN/Inf -> ORACLE_ERR_NONFINITE, nothing written but amax.
 *   2. amax = max |x|                                   (exact)
 *   3. g = RN(amax / 2688.0f)                           (2688 = 6 * 448)
 *   4. per 16-block of a row: s = E4M3_RNE_sat(RN(amax_b / RN(6 g)));
 *      RN(6 g) == 0 gives s = 0.
 *   5. D = RN(value(s) * g); code = sign(x) << 3 | e2m1_index_exact(|x|, D). */
int oracle_quantize(const void* x, int xt, int64_t rows, int64_t cols, int64_t ldx,
                    const float* gscale_in, uint8_t* codes, uint8_t* scales,
                    float* g_out, float* amax_out) {
  if (cols % 16 != 0 || rows < 0 || ldx < cols) return ORACLE_ERR_ARG;
  float amax = 0.0f;
  int nonfinite = 0;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float v = load_elem(x, xt, r * ldx + c);
      if (!isfinite(v)) nonfinite = 1;
      else if (fabsf(v) > amax) amax = fabsf(v);
    }
  if (amax_out) *amax_out = amax;
  if (nonfinite) return ORACLE_ERR_NONFINITE;

  float g;
  if (gscale_in) {
    g = *gscale_in;
    if (!isfinite(g) || g < 0.0f) return ORACLE_ERR_NONFINITE;
  } else {
    g = amax / 2688.0f;
  }
  if (g_out) *g_out = g;
  const float d6 = 6.0f * g;

  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      float blk[16];
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i) {
        blk[i] = load_elem(x, xt, r * ldx + b * 16 + i);
        if (fabsf(blk[i]) > amax_b) amax_b = fabsf(blk[i]);
      }
      uint8_t s = 0;
      if (d6 > 0.0f) {
        float s_raw = amax_b / d6;
        s = oracle_e4m3_encode(s_raw);
      }
      float D = (float)oracle_e4m3_value(s) * g;
      for (int i = 0; i < 16; i += 2) {
        uint8_t lo = (uint8_t)((signbit(blk[i]) ? 8 : 0) |
                               oracle_e2m1_index_exact(fabsf(blk[i]), D));
        uint8_t hi = (uint8_t)((signbit(blk[i + 1]) ? 8 : 0) |
                               oracle_e2m1_index_exact(fabsf(blk[i + 1]), D));
        codes[r * (cols / 2) + b * 8 + i / 2] = (uint8_t)(lo | (hi << 4));
      }
      scales[r * nb + b] = s;
    }
  }
  return ORACLE_OK;
}

/* Dequantization: y = RN(RN(e2m1 * s) * g) as float (y_f32, nullable) and its
 * bf16 RNE (y_bf16, nullable); canonical row-major codes and scales. */
void oracle_dequantize(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows,
                       int64_t cols, float* y_f32, uint16_t* y_bf16) {
  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t byte = codes[r * (cols / 2) + c / 2];
      uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      float e = (float)oracle_e2m1_value(code);
      float s = (float)oracle_e4m3_value(scales[r * nb + c / 16]);
      float p = e * s; /* exact: at most 6 significant bits, no underflow */
      float v = p * g;
      if (y_f32) y_f32[r * cols + c] = v;
      if (y_bf16) y_bf16[r * cols + c] = oracle_f32_to_bf16(v);
    }
}

/* Exact operand values e2m1 * s * g in double (what the tensor-core product
 * multiplies: e2m1 * s has <= 6 significant bits, times the 24-bit g is exact). */
void oracle_decode_f64(const uint8_t* codes, const uint8_t* scales, float g, int64_t rows,
                       int64_t cols, double* out) {
  const int64_t nb = cols / 16;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      uint8_t byte = codes[r * (cols / 2) + c / 2];
      uint8_t code = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      out[r * cols + c] =
          oracle_e2m1_value(code) * oracle_e4m3_value(scales[r * nb + c / 16]) * (double)g;
    }
}

/* Byte offset of block scale (r, j) in the tensor-core scale layout: rows in
 * tiles of 128, block columns in groups of 4, one 512-byte atom per
 * (row tile, group), atoms row-tile-major; inside an atom the 16-byte line
 * r % 32 holds rows r, r+32, r+64, r+96 (4 bytes each, one per block). */
int64_t oracle_sf_mma_offset(int64_t r, int64_t j, int64_t cols) {
  int64_t groups = (cols / 16 + 3) / 4;
  int64_t atom = (r / 128) * groups + j / 4;
  return atom * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (j % 4);
}

/* ----------------------------------------------------------- exact mean */

/* Exact sum of bf16 values.  Every finite bf16 is an integer multiple of 2^-133
 * (its smallest subnormal) of magnitude below 2^128.  Positive and negative
 * addends go to separate accumulators of 32-bit digits held in int64 (each
 * addend m * 2^sh < 2^40 lands in one digit; 2^23 addends cannot overflow). */
#define ACC_DIGITS 12
typedef struct { uint64_t d[ACC_DIGITS]; } big_t; /* base 2^32, little-endian */

static void big_normalize(big_t* a) {
  for (int i = 0; i < ACC_DIGITS - 1; ++i) {
    a->d[i + 1] += a->d[i] >> 32;
    a->d[i] &= 0xFFFFFFFFull;
  }
}

static int big_cmp(const big_t* a, const big_t* b) {
  for (int i = ACC_DIGITS - 1; i >= 0; --i) {
    if (a->d[i] != b->d[i]) return a->d[i] > b->d[i] ? 1 : -1;
  }
  return 0;
}

/* a - b for normalized a >= b */
static big_t big_sub(const big_t* a, const big_t* b) {
  big_t r;
  int64_t borrow = 0;
  for (int i = 0; i < ACC_DIGITS; ++i) {
    int64_t t = (int64_t)a->d[i] - (int64_t)b->d[i] - borrow;
    borrow = t < 0;
    r.d[i] = (uint64_t)(t + (borrow ? ((int64_t)1 << 32) : 0));
  }
  return r;
}

static int big_bit(const big_t* a, int p) {
  if (p < 0 || p >= 32 * ACC_DIGITS) return 0;
  return (int)((a->d[p / 32] >> (p % 32)) & 1u);
}

static int big_bitlen(const big_t* a) {
  for (int i = ACC_DIGITS - 1; i >= 0; --i)
    if (a->d[i]) {
      int b = 31;
      while (!((a->d[i] >> b) & 1u)) --b;
      return i * 32 + b + 1;
    }
  return 0;
}

static void big_add_bf16(big_t* pos, big_t* neg, uint16_t b) {
  int e = (b >> 7) & 0xFF, m = b & 0x7F;
  if (e == 0 && m == 0) return;
  uint64_t mant;
  int p; /* value = mant * 2^(p - 133) */
  if (e == 0) { mant = (uint64_t)m; p = 0; }            /* subnormal m * 2^-133 */
  else { mant = (uint64_t)(128 + m); p = e - 1; }       /* (128+m) * 2^(e-134) */
  big_t* a = (b & 0x8000) ? neg : pos;
  a->d[p / 32] += mant << (p % 32);
}

/* RN_f32 of (sign) * N * 2^(-133) / T for a big N and 1 <= T < 2^31, exactly:
 * Q = floor(N * 2^64 / T) by long division, then round Q with a sticky bit. */
static float round_ratio_f32(int negative, const big_t* N, uint64_t T) {
  if (big_bitlen(N) == 0) return 0.0f;
  big_t S = {{0}};
  for (int i = 0; i + 2 < ACC_DIGITS; ++i) S.d[i + 2] = N->d[i]; /* N * 2^64 */
  big_t Q = {{0}};
  uint64_t rem = 0;
  for (int i = ACC_DIGITS - 1; i >= 0; --i) {
    uint64_t cur = (rem << 32) | S.d[i];
    Q.d[i] = cur / T;
    rem = cur % T;
  }
  const int scale = 133 + 64; /* value = Q * 2^-scale (+ rem/T below the LSB) */
  int L = big_bitlen(&Q);
  int E = (L - 1) - scale; /* exponent of the leading bit */
  int lsb = E - 23;
  if (lsb < -149) lsb = -149; /* binary32 subnormal grid */
  int shift = lsb + scale;    /* bits of Q below the kept LSB */
  uint64_t mant = 0;
  for (int p = L - 1; p >= shift && p >= 0; --p) mant = (mant << 1) | (uint64_t)big_bit(&Q, p);
  int guard = big_bit(&Q, shift - 1);
  int sticky = rem != 0;
  for (int p = shift - 2; p >= 0 && !sticky; --p) sticky |= big_bit(&Q, p);
  if (guard && (sticky || (mant & 1u))) ++mant;
  double v = ldexp((double)mant, lsb); /* exact: mant <= 2^24 */
  float f = (float)v;
  return negative ? -f : f;
}

/* mu = RN_f32(exact sum of the `T` bf16 values x[t * stride] / T). */
float oracle_exact_mean_bf16(const uint16_t* x, int64_t T, int64_t stride) {
  big_t pos = {{0}}, neg = {{0}};
  for (int64_t t = 0; t < T; ++t) big_add_bf16(&pos, &neg, x[t * stride]);
  big_normalize(&pos);
  big_normalize(&neg);
  int c = big_cmp(&pos, &neg);
  if (c == 0) return 0.0f;
  big_t mag = c > 0 ? big_sub(&pos, &neg) : big_sub(&neg, &pos);
  return round_ratio_f32(c < 0, &mag, (uint64_t)T);
}

/* ----------------------------------------------------------- KV cache */

/* One chunk append.  k, v: bf16 bits [T][H][Dh].  [TW §四]
 *   mu[h*Dh+d] = RN(exact_sum_t k[t,h,d] / T)   (per head, per dim, over the chunk)
 *   K'[t,h,d]  = RN(k - mu)                     (FP32)
 *   K', V each quantized as one tensor of T*H rows and Dh columns (blocks of 16
 *   along head_dim, one tensor scale per chunk), i.e. oracle_quantize. */
int oracle_kv_append(const uint16_t* k, const uint16_t* v, int64_t T, int64_t H, int64_t Dh,
                     float* mu, float* g_k, float* g_v, uint8_t* k_codes, uint8_t* k_scales,
                     uint8_t* v_codes, uint8_t* v_scales, float* amax_k, float* amax_v) {
  const int64_t C = H * Dh;
  for (int64_t i = 0; i < T * C; ++i) {
    if (!isfinite(oracle_bf16_to_f32(k[i])) || !isfinite(oracle_bf16_to_f32(v[i])))
      return ORACLE_ERR_NONFINITE;
  }
  for (int64_t c = 0; c < C; ++c) mu[c] = oracle_exact_mean_bf16(k + c, T, C);
  float* kp = (float*)malloc(sizeof(float) * (size_t)(T * C));
  if (!kp) return ORACLE_ERR_ARG;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < C; ++c) kp[t * C + c] = oracle_bf16_to_f32(k[t * C + c]) - mu[c];
  int rc = oracle_quantize(kp, 1, T * H, Dh, Dh, NULL, k_codes, k_scales, g_k, amax_k);
  free(kp);
  if (rc) return rc;
  return oracle_quantize(v, 0, T * H, Dh, Dh, NULL, v_codes, v_scales, g_v, amax_v);
}

/* Dequantization of one chunk for a window:
 *   K^ = bf16(RN(RN(RN(e2m1 * s) * g_K) + mu)),  V^ = bf16(RN(RN(e2m1 * s) * g_V)).
 * The K step is a separate multiply and add (no fused multiply-add). */
void oracle_kv_dequant_chunk(const uint8_t* k_codes, const uint8_t* k_scales,
                             const uint8_t* v_codes, const uint8_t* v_scales, const float* mu,
                             float g_k, float g_v, int64_t T, int64_t H, int64_t Dh,
                             uint16_t* k_out, uint16_t* v_out) {
  const int64_t C = H * Dh;
  float* tmp = (float*)malloc(sizeof(float) * (size_t)(T * C));
  if (!tmp) return;
  oracle_dequantize(k_codes, k_scales, g_k, T * H, Dh, tmp, NULL);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < C; ++c) {
      float s = tmp[t * C + c] + mu[c];
      k_out[t * C + c] = oracle_f32_to_bf16(s);
    }
  free(tmp);
  oracle_dequantize(v_codes, v_scales, g_v, T * H, Dh, NULL, v_out);
}

/* ----------------------------------------------------------- activation */

/* GELU, tanh form (Hendrycks & Gimpel), in double:
 *   h = 0.5 c (1 + tanh(u)),  u = sqrt(2/pi) (c + 0.044715 c^3),
 * evaluated through the exact identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)), i.e.
 * h = c / (1 + exp(-2u)).  Written as 1 + tanh(u), the sum cancels for u << 0 (tanh
 * is -1 to within its rounding error), which leaves no correct digit in the negative
 * tail; the quotient form keeps the relative error at a few ulp everywhere. */
double oracle_gelu_tanh(double c) {
  const double k = sqrt(2.0 / 3.14159265358979323846);
  const double u = k * (c + 0.044715 * c * c * c);
  return c / (1.0 + exp(-2.0 * u));
}

void oracle_gelu_tanh_array(const float* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_gelu_tanh((double)c[i]);
}

/* ---------------------------------------------------------------- LoRA merge */

/* A LoRA update merged into a weight before the weight is quantized.
 * [ZD] github.zuobiaodaohang.com, "长视频生成的两堵物理墙", section "NVFP4：数据体积砍到
 * 1/4", further optimizations: "LoRA before quantization" (the LoRA is loaded into
 * the weight first, then the weight is quantized, for accuracy).
 * Reading (the page gives no formula): the usual LoRA update
 *   W' = W + scale * (B A),  B [rows, rank], A [rank, cols],
 * in binary32 with one fixed order of operations:
 *   acc = 0;  for j = 0 .. rank-1:  acc = RN(acc + RN(B[r][j] * A[j][c]));
 *   W'[r][c] = RN(W[r][c] + RN(scale * acc)).
 * W is bf16 bits (wt 0) or float (wt 1), row pitch ldw elements; B has row pitch
 * rank, A row pitch cols; out is float [rows, cols] with row pitch ldo.  Non-finite
 * values propagate (quantizing the result reports them). */
void oracle_lora_merge(const void* w, int wt, int64_t rows, int64_t cols, int64_t ldw, const float* b,
                       const float* a, int64_t rank, float scale, float* out, int64_t ldo) {
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      float acc = 0.0f;
      for (int64_t j = 0; j < rank; ++j) {
        const float p = b[r * rank + j] * a[j * cols + c];
        acc = acc + p;
      }
      const float u = scale * acc;
      out[r * ldo + c] = load_elem(w, wt, r * ldw + c) + u;
    }
  }
}

/* ------------------------------------------------------- amax history (C8) */

/* Tensor scale of a requantizing GEMM epilogue from the max|h| of earlier calls.
 * The epilogue quantizes before its own max|h| is known, so it takes a supplied
 * scale; reading fixed here: keep the last len values of max|h| (newest first)
 * and supply g = RN(max(history) / 2688), the tensor-scale formula of quantize.
 * Push: history[i] = history[i-1] for i = len-1 .. 1, history[0] = amax_new, then
 * *g_out from the updated history.  A non-finite amax_new changes nothing and
 * returns ORACLE_ERR_NONFINITE. */
int oracle_amax_history_push(float* history, int64_t len, float amax_new, float* g_out) {
  if (!(fabsf(amax_new) <= 3.402823466e38f)) return ORACLE_ERR_NONFINITE;
  for (int64_t i = len - 1; i >= 1; --i) history[i] = history[i - 1];
  history[0] = amax_new;
  float m = 0.0f;
  for (int64_t i = 0; i < len; ++i)
    if (history[i] > m) m = history[i];
  *g_out = m / 2688.0f;
  return ORACLE_OK;
}
