// lora.cu — a LoRA update merged into a weight before the weight is quantized.
//
// github.zuobiaodaohang.com, "长视频生成的两堵物理墙", section "NVFP4：数据体积砍到 1/4",
// further optimizations: "LoRA before quantization" — the LoRA is loaded into the
// weight first and the weight is quantized afterwards.
//
// Reading fixed here (the page gives no formula): W' = W + scale * (B A) in binary32
// with one fixed order, acc = RN(acc + RN(B[r][j] * A[j][c])) for j = 0 .. rank-1,
// then W' = RN(W + RN(scale * acc)); nvfp4_quantize then quantizes W' (FP32 input).
// The explicit __fmul_rn / __fadd_rn keep that order free of fused multiply-adds.
//
// Tiling: a CTA computes 16 rows x 128 columns; the rank is walked in steps of 32
// with B (transposed, so a thread's 8 rows are 2 vector loads) and A staged in
// shared memory.  Thread t owns column t % 128 and rows 8 (t / 128) .. + 7.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kRows = 16, kCols = 128, kStep = 32, kThreads = 256;

struct LoraParams {
  const uint8_t* w;
  bool w_bf16;
  int64_t rows, cols, ldw;
  const float* b;  // [rows][rank]
  const float* a;  // [rank][cols]
  int64_t rank;
  float scale;
  float* out;
  int64_t ldo;
};

__global__ void __launch_bounds__(kThreads) lora_merge_kernel(LoraParams p) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float bs[kStep][kRows];  // bs[j][row]
  __shared__ float as[kStep][kCols];
  const int64_t r0 = (int64_t)blockIdx.y * kRows, c0 = (int64_t)blockIdx.x * kCols;
  const int tc = threadIdx.x % kCols, tr = (threadIdx.x / kCols) * 8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
  for (int64_t j0 = 0; j0 < p.rank; j0 += kStep) {
    const int nj = (int)min((int64_t)kStep, p.rank - j0);
    for (int e = threadIdx.x; e < kStep * kRows; e += kThreads) {
      const int jj = e % kStep, rr = e / kStep;
      const int64_t r = r0 + rr;
      bs[jj][rr] = (jj < nj && r < p.rows) ? p.b[r * p.rank + j0 + jj] : 0.0f;
    }
    for (int e = threadIdx.x; e < kStep * kCols; e += kThreads) {
      const int jj = e / kCols, cc = e % kCols;
      const int64_t c = c0 + cc;
      as[jj][cc] = (jj < nj && c < p.cols) ? p.a[(j0 + jj) * p.cols + c] : 0.0f;
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      const float av = as[jj][tc];
      const float4 b0 = *reinterpret_cast<const float4*>(&bs[jj][tr]);
      const float4 b1 = *reinterpret_cast<const float4*>(&bs[jj][tr + 4]);
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(bv[i], av));
    }
    __syncthreads();
  }
  const int64_t c = c0 + tc;
  if (c >= p.cols) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = r0 + tr + i;
    if (r >= p.rows) break;
    const float w = p.w_bf16 ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(p.w)[r * p.ldw + c] << 16)
                             : reinterpret_cast<const float*>(p.w)[r * p.ldw + c];
    p.out[r * p.ldo + c] = __fadd_rn(w, __fmul_rn(p.scale, acc[i]));
  }
}

}  // namespace

cudaError_t launch_lora_merge(const LoraArgs& a, cudaStream_t s) {
  if (a.rows == 0 || a.cols == 0) return cudaSuccess;
  LoraParams p;
  p.w = static_cast<const uint8_t*>(a.w);
  p.w_bf16 = a.w_bf16;
  p.rows = a.rows;
  p.cols = a.cols;
  p.ldw = a.ldw;
  p.b = a.b;
  p.a = a.a;
  p.rank = a.rank;
  p.scale = a.scale;
  p.out = a.out;
  p.ldo = a.ldo;
  dim3 grid((unsigned)((a.cols + kCols - 1) / kCols), (unsigned)((a.rows + kRows - 1) / kRows));
  launch_pdl(lora_merge_kernel, grid, kThreads, 0, s, p);
  return cudaGetLastError();
}

}  // namespace nvfp4
