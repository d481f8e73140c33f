// gemm.cu — W4A4 block-scaled GEMM on the sm_100a tensor cores.
//
// techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存", §四:
// all matmuls of the model run with 4-bit weights and activations; they are the
// dominant cost of generation.  ai-manual.ru, "LongLive-2.0 ...", section
// "Как это работает под капотом": scaling and quantization are merged into one
// kernel — here the NVFP4 requantization of the activated output runs in the GEMM
// epilogue.
//
//   c[m, n] = RN(acc[m, n] * RN(gA * gW)),   C = act(c)  (act: none or GELU-tanh)
//   acc     = sum_k (e2m1(A[m,k]) sA[m,k/16]) (e2m1(W[n,k]) sW[n,k/16])  (FP32, tensor core)
//
// Two kernels.  gemm_kernel (below): one persistent CTA per SM, 128 x 128 tiles,
// 14 warps.  gemm_pair_kernel (further down): CTA pairs, 256 x 256 tiles, 24 warps.
// Structure of gemm_kernel:
//   warp 0      TMA producer: A and W code tiles (128 B swizzle, 128 rows x 256
//               values per stage) and the stage's scale atoms (bulk copies).
//   warp 1      MMA issuer: tcgen05.mma.kind::mxf4nvf4.block_scale (UE4M3,
//               16-value blocks, K = 64 per instruction) into tensor memory.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (one row per thread,
//               two warps per 32-lane quarter, each taking half the columns),
//               scaling, optional GELU and NVFP4 requantization, stores.
//   warps 10..13 scale factors: each warp copies the stage's scale atoms from
//               shared memory into its 32-lane quarter of tensor memory with
//               tcgen05.st (the 4-way lane replication the block-scaled MMA reads).
//               Doing this on the SM's load/store path keeps it off the tensor
//               pipe, where tcgen05.cp copies serialize with the MMAs.
// Two accumulator buffers in tensor memory let the epilogue of one tile overlap
// the main loop of the next.  No TMA load uses cluster multicast.
//
// Every wait is bounded: after ~2 s a wait records NVFP4_ERR_TIMEOUT in the
// status word, raises a CTA-wide abort flag and the CTA drains its own
// asynchronous work (bounded again) before it frees tensor memory and exits.
#include <cuda.h>

#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nvfp4 {
namespace {

using namespace tc;

constexpr int kBM = 128;           // tile rows (A rows, TMEM lanes)
constexpr int kBN = 128;           // tile columns (W rows)
constexpr int kBKBytes = 128;      // per stage: 128 bytes of packed codes = 256 values
constexpr int kKPerMma = 64;       // values per tcgen05.mma (32 bytes)
constexpr int kStages = 4;
constexpr int kAccStages = 2;
constexpr int kEpiWarps = 8;      // two per 32-lane quarter of tensor memory
constexpr int kThreads = 32 * (2 + kEpiWarps + 4);  // 14 warps
constexpr int kEpiWarp0 = 2;      // warps 2..9: epilogue
constexpr int kSfWarp0 = kEpiWarp0 + kEpiWarps;  // warps 10..13: scale factors to tensor memory
constexpr int kTmemCols = 512;
constexpr int kSfColBase = kAccStages * kBN;  // scale-factor columns follow the accumulators

constexpr int kABytes = kBM * kBKBytes;        // 16 KB
constexpr int kBBytes = kBN * kBKBytes;        // 16 KB
constexpr int kSfaBytes = (kBM / 128) * 4 * 512;  // 4 atoms (one per 64-value group)
constexpr int kSfbBytes = (kBN / 128) * 4 * 512;
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
// Output staging for TMA stores: per epilogue warp two 32-row x 128-byte buffers.
constexpr int kStagingBytesPerWarp = 2 * 32 * 128;
constexpr int kStagingBytes = kEpiWarps * kStagingBytesPerWarp;
constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 /*barriers*/ + 1024 /*alignment*/;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Test hook for the bounded waits (set only by nvfp4_debug_gemm_fault).
std::atomic<unsigned long long> g_debug_wait_limit_ns{0};
std::atomic<int> g_debug_drop_first_stage{0};

struct Params {
  int64_t M, N, K;
  int64_t num_m, num_n, num_k64;  // tiles along M, N and 64-value groups along K
  int64_t num_tiles;
  int64_t sfa_row_tile_bytes;     // bytes of scale atoms per 128-row tile of A
  int64_t sfw_row_tile_bytes;
  const uint8_t* sfa;
  const uint8_t* sfw;
  const float* ga;
  const float* gw;
  uint8_t* c;
  bool c_bf16;
  int64_t ldc;
  int act;
  uint8_t* q_codes;
  int64_t q_ld_codes;
  uint8_t* q_scales;
  int64_t q_groups;
  const float* q_gscale_in;
  float* q_gscale_out;
  float* q_amax_out;
  float* h_out;
  unsigned* status;
  unsigned long long wait_limit_ns;
  int drop_first_stage;  // test hook: skip the first stage's loads (the waits for it run out)
};

// ----------------------------------------------------------------- PTX helpers
// (mbarriers with bounded waits, TMA tile loads and stores, descriptors: tc.cuh)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Instruction descriptor of kind::mxf4nvf4 with UE4M3 scales: A and B E2M1
// (format 1 at bits 7..9 and 10..12), both K-major, N >> 3 at bits 17..22,
// scale format 0 (UE4M3) at bit 23, M >> 4 at bits 24..28, dense K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ void mma_mxf4nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's lane (warp-collective).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
      "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, uint4 v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// max(a, b) that returns NaN when either operand is NaN
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// GELU, tanh form: 0.5 c (1 + tanh(u)) with u = sqrt(2/pi) (c + 0.044715 c^3),
// evaluated through the identity 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)):
//   h = c / (1 + 2^x),  x = -2 u log2(e) = c (A c^2 + B),
//   B = -2 sqrt(2/pi) log2(e), A = 0.044715 B,
// with the hardware exp2 and reciprocal approximations (relative error ~2^-22 over
// the binary32 range, inside the 2^-20 (|c| + |h|) the parity tests hold h to; large
// |c| gives h = c or -0, infinities as the formula).  No paired multiply here feeds a
// paired add, so no step can be contracted into a fused multiply-add.
// Two values at a time: the FP32 steps as two-lane operations (same roundings as the
// scalar form), exp2 and reciprocal per value.
__device__ __forceinline__ void gelu_tanh2(float& c0, float& c1) {
  float t0, t1, u0, u1, x0, x1, e0, e1, d0, d1, r0, r1;
  mul2(t0, t1, c0, c1, c0, c1);
  fma2(u0, u1, t0, t1, -0.1029432396f, -0.1029432396f, -2.3022081983f, -2.3022081983f);
  mul2(x0, x1, c0, c1, u0, u1);
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(x0));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(x1));
  add2(d0, d1, 1.0f, 1.0f, e0, e1);
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(d0));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(d1));
  mul2(c0, c1, c0, c1, r0, r1);
}

// ----------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
                const __grid_constant__ CUtensorMap map_c, Params p) {
  pdl_trigger();  // the next kernel on the stream may start its set-up
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kStages * kStageBytes;  // 1024-aligned
  uint8_t* bar_area = staging + kStagingBytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty_bar = full_bar + kStages;
  uint64_t* tfull_bar = empty_bar + kStages;
  uint64_t* tempty_bar = tfull_bar + kAccStages;
  uint64_t* sf_bar = tempty_bar + kAccStages;  // [kStages] scale factors in tensor memory
  uint64_t* done_bar = sf_bar + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < kAccStages; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), kEpiWarps * 32);
    }
    for (int st = 0; st < kStages; ++st) mbar_init(smem_u32(&sf_bar[st]), 4);
    mbar_init(smem_u32(done_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // operands and scales were written by earlier kernels
  const unsigned long long limit = p.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
      const int64_t kstages = (p.num_k64 + 3) / 4;
      uint32_t it = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        const int64_t mt = tile % p.num_m, nt = tile / p.num_m;
        for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          if (p.drop_first_stage && it == 0) continue;  // its full barrier never completes
          const int64_t g0 = ks * 4;
          const int nvalid = (int)min((int64_t)4, p.num_k64 - g0);
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t fb = smem_u32(&full_bar[s]);
          mbar_arrive_expect_tx(fb, kABytes + kBBytes + 2 * nvalid * 512);
          tma_load_2d(smem_u32(st), &map_a, fb, (int32_t)(ks * kBKBytes), (int32_t)(mt * kBM));
          tma_load_2d(smem_u32(st + kABytes), &map_w, fb, (int32_t)(ks * kBKBytes), (int32_t)(nt * kBN));
          bulk_load(smem_u32(st + kABytes + kBBytes), p.sfa + mt * p.sfa_row_tile_bytes + g0 * 512,
                    nvalid * 512, fb);
          bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes),
                    p.sfw + nt * p.sfw_row_tile_bytes + g0 * 512, nvalid * 512, fb);
        }
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      // drain: every load this thread issued must land before the CTA exits
      const uint32_t n_issued = it;
      for (uint32_t j = (n_issued > (uint32_t)kStages ? n_issued - kStages : 0); j < n_issued; ++j) {
        const int s = j % kStages;
        mbar_wait_drain(smem_u32(&full_bar[s]), (j / kStages) & 1u, limit);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int64_t kstages = (p.num_k64 + 3) / 4;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tcount) {
        const int a = tcount % kAccStages;
        const uint32_t aph = (tcount / kAccStages) & 1u;
        if (!mbar_wait(smem_u32(&tempty_bar[a]), aph ^ 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t d_tmem = tmem_base + a * kBN;
        for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          // the scale warps saw this stage's TMA land and put its scales in tensor memory
          if (!mbar_wait(smem_u32(&sf_bar[s]), ph, abort_flag, limit)) {
            ok = false;
            break;
          }
          fence_after();
          const int nvalid = (int)min((int64_t)4, p.num_k64 - ks * 4);
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t a_addr = smem_u32(st), b_addr = smem_u32(st + kABytes);
          for (int k = 0; k < nvalid; ++k) {
            const uint32_t sf_col = tmem_base + kSfColBase + (s * 4 + k) * 8;
            const uint64_t adesc = smem_desc(a_addr + k * 32, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(b_addr + k * 32, 16, 1024, 2);
            mma_mxf4nvf4(d_tmem, adesc, bdesc, sf_col, sf_col + 4, (ks > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty_bar[s]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull_bar[a]));
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      // drain: all MMAs this thread issued complete before tensor memory is freed
      mma_commit(smem_u32(done_bar));
      mbar_wait_drain(smem_u32(done_bar), 0, limit);
    }
  } else if (warp >= kSfWarp0) {
    // ------------------------------------------------------------ scale factors
    // Tensor-memory scale layout of the block-scaled MMA: for MMA k of stage s,
    // columns c = kSfColBase + (s*4 + k)*8 hold A's scales (c .. c+3) and W's
    // (c+4 .. c+7); lane l of EVERY 32-lane quarter holds, in column c + j, the 4
    // block scales of row l + 32 j.  A 512-byte scale atom in shared memory has
    // exactly that content in its 16-byte line l, so lane l of each quarter loads
    // line l of the 4 atoms of A and of W and stores them as 32 columns.
    const int quarter = warp & 3;
    const int64_t kstages = (p.num_k64 + 3) / 4;
    uint32_t it = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full_bar[s]), ph, abort_flag, limit))) {
          ok = false;
          break;
        }
        const int nvalid = (int)min((int64_t)4, p.num_k64 - ks * 4);
        const uint8_t* sfa = smem + s * kStageBytes + kABytes + kBBytes;
        const uint8_t* sfb = sfa + kSfaBytes;
        uint32_t r[32];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
          if (k < nvalid) {
            a = *reinterpret_cast<const uint4*>(sfa + k * 512 + lane * 16);
            b = *reinterpret_cast<const uint4*>(sfb + k * 512 + lane * 16);
          }
          r[8 * k + 0] = a.x; r[8 * k + 1] = a.y; r[8 * k + 2] = a.z; r[8 * k + 3] = a.w;
          r[8 * k + 4] = b.x; r[8 * k + 5] = b.y; r[8 * k + 6] = b.z; r[8 * k + 7] = b.w;
        }
        tmem_st_32x32b_x32(tmem_base + ((uint32_t)(quarter * 32) << 16) + kSfColBase + s * 32, r);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sf_bar[s]));
      }
    }
    if (!ok) {
      if (lane == 0) set_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    const int col_half = (warp - kEpiWarp0) / 4;  // columns [64 col_half, 64 col_half + 64) of a tile
    const int row_in_tile = quarter * 32 + lane;
    const float gab = (*p.ga) * (*p.gw);
    float gq = 0.0f, d6q = 0.0f, r6q = 0.0f;
    if (p.q_codes) {
      gq = *p.q_gscale_in;
      d6q = 6.0f * gq;
      r6q = 1.0f / d6q;
      if (blockIdx.x == 0 && threadIdx.x == kEpiWarp0 * 32) *p.q_gscale_out = gq;
    }
    unsigned amax_bits = 0;
    uint32_t tcount = 0, chunk = 0;
    for (int64_t tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tcount) {
      const int a = tcount % kAccStages;
      const uint32_t aph = (tcount / kAccStages) & 1u;
      // warp-uniform outcome: the tensor-memory loads below are warp-collective
      const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&tfull_bar[a]), aph, abort_flag, limit));
      if (!got) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      fence_after();
      const int64_t mt = tile % p.num_m, nt = tile / p.num_m;
      const int64_t row = mt * kBM + row_in_tile;
      const bool row_ok = row < p.M;
      for (int cc = col_half * (kBN / 2); cc < (col_half + 1) * (kBN / 2); cc += 32) {
        uint32_t r[32];
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + a * kBN + cc;
        tmem_ld_32x32b_x32(taddr, r);
        const int64_t col0 = nt * kBN + cc;
        if (col0 >= p.N) continue;  // warp-uniform
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          mul2(v[i], v[i + 1], __uint_as_float(r[i]), __uint_as_float(r[i + 1]), gab, gab);
        if (p.act == 1) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) gelu_tanh2(v[i], v[i + 1]);
        }
        if (p.c) {
          // Stage this warp's 32 rows x 32 columns in shared memory (swizzled like the
          // tensor map, so the writes are bank-conflict free) and store the box with
          // one TMA store: full-line global writes, rows >= M / columns >= N clipped.
          const uint32_t buf = smem_u32(staging) + (uint32_t)((warp - kEpiWarp0) * kStagingBytesPerWarp) +
                               (uint32_t)((chunk & 1) * 4096);
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
          if (p.c_bf16) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              st_shared_v4(buf + lane * 64 + ((u ^ ((lane >> 1) & 3)) * 16),
                           make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                      pack_bf16x2(v[8 * u + 4], v[8 * u + 5]),
                                      pack_bf16x2(v[8 * u + 6], v[8 * u + 7])));
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u)
              st_shared_v4(buf + lane * 128 + ((u ^ (lane & 7)) * 16),
                           make_uint4(__float_as_uint(v[4 * u]), __float_as_uint(v[4 * u + 1]),
                                      __float_as_uint(v[4 * u + 2]), __float_as_uint(v[4 * u + 3])));
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_c, buf, (int32_t)col0, (int32_t)(mt * kBM + quarter * 32));
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
          ++chunk;
        }
        if (!row_ok) {
          if (p.q_codes) {
            // zero the scale padding of rows beyond M so the next GEMM reads finite scales
            if (row < (p.M + 127) / 128 * 128)
              *reinterpret_cast<uint16_t*>(p.q_scales + sf_mma_offset(row, col0 / 16, p.q_groups)) = 0;
          }
          continue;
        }
        const int nvc = (int)min((int64_t)32, p.N - col0);  // 16 on a ragged last chunk
        if (p.h_out) {
          float* hd = p.h_out + row * p.N + col0;
          if (nvc == 32) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              stg_v4(hd + 4 * q, make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                            __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3])));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nvc) hd[i] = v[i];
          }
        }
        if (p.q_amax_out && !p.q_codes) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nvc) amax_bits = max(amax_bits, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        }
        if (p.q_codes) {  // N % 64 == 0 here, so the chunk is whole
          uint32_t w[4];
          uint32_t sc[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float s0[8], s1[8];
            // block max of |h|, NaN-propagating: a NaN makes the block's scale the
            // E4M3 NaN and (above +inf as bits) max|h| for q_amax_out non-finite
            float amax_b = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax_b = fmax_nan(amax_b, fabsf(v[16 * b + k]));
            amax_bits = max(amax_bits, __float_as_uint(amax_b));
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              s0[k] = v[16 * b + k];
              s1[k] = v[16 * b + 8 + k];
            }
            const uint32_t s = block_scale_fast(amax_b, d6q, r6q);
            const BlockEncoder enc(e4m3_to_float(s) * gq);
            w[2 * b] = enc.encode8s(s0);
            w[2 * b + 1] = enc.encode8s(s1);
            sc[b] = s;
          }
          stg_v4(p.q_codes + row * p.q_ld_codes + col0 / 2, make_uint4(w[0], w[1], w[2], w[3]));
          *reinterpret_cast<uint16_t*>(p.q_scales + sf_mma_offset(row, col0 / 16, p.q_groups)) =
              (uint16_t)(sc[0] | (sc[1] << 8));
        }
      }
      fence_before();
      mbar_arrive(smem_u32(&tempty_bar[a]));
    }
    if (p.q_amax_out) {
      amax_bits = warp_max_u32(amax_bits);
      if (lane == 0 && amax_bits) atomicMax(reinterpret_cast<unsigned*>(p.q_amax_out), amax_bits);
    }
    // every TMA store of this warp has finished before the CTA exits
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ============================================================ 2-CTA pair kernel
// One cluster of 2 CTAs computes a 256 x kBN tile (kBN = 256) with
// tcgen05.mma.cta_group::2 (M = 256, N = kBN, K = 64 per instruction): CTA r of the
// pair holds rows [128 r, 128 r + 128) of the A tile and rows [r kBN/2, (r + 1) kBN/2)
// of the W tile in its shared memory, and rows 128 r .. of the accumulator in its
// tensor memory.  The even CTA issues every MMA; operands are read from both CTAs'
// shared memory by the hardware.  Each CTA loads only its own halves (no TMA
// multicast): 32 KB of codes per 256 K values per CTA for a 128 x 256 share of the
// output, against 48 KB for a 128 x 256 tile of one CTA.
//
// Tensor memory per CTA (512 columns): kAccStages accumulators of kBN columns (one
// at kBN = 256), then one scale slot per pipeline stage of 4 MMAs x (4 + 4 kWTiles)
// columns: per MMA [A scales | W scales of each 128-row W tile]; the W scales of all
// kBN rows are present in both CTAs (the hardware reads them in the SM that holds
// the accumulator rows).
namespace pair {

constexpr int kBM = 256;            // rows per pair tile (128 per CTA)
constexpr int kBN = 256;            // columns per pair tile: 128 or 256
constexpr int kBNHalf = kBN / 2;    // W rows per CTA
constexpr int kWTiles = kBN / 128;  // 128-row W scale tiles per pair tile
constexpr int kStages = 5;
constexpr int kSfSlots = kStages;  // one per pipeline stage
constexpr int kAccStages = kBN == 256 ? 1 : 2;
// Warp roles, in 4-warp groups (the unit of register reallocation):
//   warpgroup 0  warp 0 TMA producer, warp 1 MMA issuer (leader CTA), warps 2-3 idle
//   warpgroup 1  warps 4..7 scale factors, one per tensor-memory lane quarter
//   2..5         warps 8..23 epilogue, 4 per lane quarter, 64 columns each
constexpr int kEpiWarps = 16;
constexpr int kSfWarp0 = 4;
constexpr int kEpiWarp0 = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);  // 768
// Registers: the kernel is launched with kRegsLaunch a thread (24 warps, six on each
// of the SM's four 16K-register files: 16384 / 192 = 85, allocated in steps of 8).
// Warpgroups 0 and 1 then release registers with setmaxnreg.dec and the four
// epilogue warpgroups take them with setmaxnreg.inc; an increase waits until the
// released registers cover it, so the split must balance exactly (the host checks
// the compiled launch count before the first launch).
constexpr int kRegsLaunch = 80;
constexpr int kRegsCtl = 40;   // warpgroup 0 (fewer make the MMA loop spill)
constexpr int kRegsSf = 24;    // warpgroup 1
constexpr int kRegsEpi = 104;  // warpgroups 2..5: 64 accumulator values a thread + work
static_assert(4 * (kRegsEpi - kRegsLaunch) <= (kRegsLaunch - kRegsCtl) + (kRegsLaunch - kRegsSf),
              "the epilogue's extra registers must come from warpgroups 0 and 1");
static_assert(kRegsCtl % 8 == 0 && kRegsSf % 8 == 0 && kRegsEpi % 8 == 0 && kRegsCtl >= 24 && kRegsSf >= 24 &&
                  kRegsCtl <= kRegsLaunch && kRegsSf <= kRegsLaunch && kRegsEpi >= kRegsLaunch,
              "setmaxnreg counts");
constexpr int kABytes = 128 * kBKBytes;           // 16 KB
constexpr int kBBytes = kBNHalf * kBKBytes;       // 8 or 16 KB
constexpr int kSfaBytes = 4 * 512;                // own 128 rows, 4 groups
constexpr int kSfbBytes = kWTiles * 4 * 512;      // all kBN W rows of the tile x 4 groups
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
// Output staging: 32 rows x 64 bytes per epilogue warp.  A bf16 output box is one
// warp's buffer; an FP32 box (128 rows x 16 columns) is the 4 buffers of a column
// group, contiguous because the group's warps are consecutive.
constexpr int kStagingBytesPerWarp = 32 * 64;
constexpr int kStagingBytes = kEpiWarps * kStagingBytesPerWarp;
constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kBN == 4 * 64, "epilogue warps cover 64 columns each");
constexpr int kSfColBase = kAccStages * kBN;      // 256
constexpr int kSfPerMma = 4 + 4 * kWTiles;      // A's 4 columns, then 4 per W scale tile
constexpr int kSfSlotCols = 4 * kSfPerMma;
static_assert(kSfColBase + kSfSlots * kSfSlotCols <= 512, "tensor memory budget");
static_assert(kBN == 128 || kBN == 256, "pair tile width");
// kind::mxf4nvf4, E2M1 x E2M1, UE4M3 scales, K-major, N = kBN, M = 256
constexpr uint32_t kIdesc2 = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <int kRegs>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <int kRegs>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// address of the same shared-memory variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on a barrier of another CTA of the cluster.  What it orders is tensor
// memory traffic, which the tcgen05 fences around the arrive and the wait order;
// no cluster-scope memory fence is needed (and one costs a membar per arrive).
// AND of `ok` over the 128 threads (4 warps) that use named barrier `id`; every
// one of them must call it.
__device__ __forceinline__ bool group_all(uint32_t id, bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred q, p;\n setp.ne.u32 q, %1, 0;\n bar.red.and.pred p, %2, 128, q;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void mma2(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t sfa, uint32_t sfb,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// arrive on the barrier at this shared-memory offset in every CTA of `mask`
// once all previously issued MMAs of this thread have completed
__device__ __forceinline__ void commit2(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

struct Params2 {
  int64_t M, N, K;
  int64_t num_m, num_n, num_k64, num_tiles;
  int64_t a_row_tiles, w_row_tiles;  // 128-row scale tiles present in each scale buffer
  int64_t sf_row_tile_bytes;         // num_k64 * 512
  const uint8_t* sfa;
  const uint8_t* sfw;
  const float* ga;
  const float* gw;
  bool has_c, c_bf16;
  int act;
  uint8_t* q_codes;
  int64_t q_ld_codes;
  uint8_t* q_scales;
  int64_t q_groups;
  const float* q_gscale_in;
  float* q_gscale_out;
  float* q_amax_out;
  float* h_out;
  unsigned* status;
  unsigned long long wait_limit_ns;
  int drop_first_stage;  // test hook: skip the first stage's loads (the waits for it run out)
};

// kFused = false: plain FP32/bf16 output.  kFused = true: the general epilogue
// (GELU, h_out, max|h|, NVFP4 requantization, optional C).
template <bool kFused>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_c, Params2 p) {
  pdl_trigger();  // the next kernel on the stream may start its set-up
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kStages * kStageBytes;
  uint8_t* bar_area = staging + kStagingBytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(bar_area);   // own TMA landed
  uint64_t* empty_bar = full_bar + kStages;                      // MMAs of the stage done (both CTAs)
  uint64_t* sf_bar = empty_bar + kStages;                        // leader: scales of both CTAs in TMEM
  uint64_t* tfull_bar = sf_bar + kStages;                        // accumulator ready (both CTAs)
  uint64_t* tempty_bar = tfull_bar + kAccStages;                 // leader: both epilogues drained
  uint64_t* done_bar = tempty_bar + kAccStages;                  // leader: all MMAs complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
      mbar_init(smem_u32(&sf_bar[s]), 2 * 4);
    }
    for (int a = 0; a < kAccStages; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(done_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  cluster_sync();  // barriers of both CTAs initialized, tensor memory allocated
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // operands and scales were written by earlier kernels
  const unsigned long long limit = p.wait_limit_ns;
  const int64_t kstages = (p.num_k64 + 3) / 4;

  if (warp < kSfWarp0) {
    // warpgroup 0: producer (warp 0), MMA issuer (warp 1); warps 2 and 3 idle
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      if (lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
        uint32_t it = 0;
        bool ok = true;
        for (int64_t tile = pair; tile < p.num_tiles && ok; tile += num_pairs) {
          const int64_t mt = tile % p.num_m, nt = tile / p.num_m;
          const int64_t a_rt = mt * 2 + rank;                 // this CTA's 128-row tile of A
          const bool has_sfa = a_rt < p.a_row_tiles;
          const int64_t n0 = nt * kBN;
          const int64_t w_rt = n0 / 128;  // first 128-row W scale tile of the pair tile
          int w_tiles = 0;                // W scale tiles present (the last pair tile may be ragged)
          for (int t = 0; t < kWTiles; ++t) w_tiles += (w_rt + t < p.w_row_tiles) ? 1 : 0;
          for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, abort_flag, limit)) {
              ok = false;
              break;
            }
            if (p.drop_first_stage && it == 0) continue;  // its full barrier never completes
            const int64_t g0 = ks * 4;
            const int nvalid = (int)min((int64_t)4, p.num_k64 - g0);
            uint8_t* st = smem + s * kStageBytes;
            const uint32_t fb = smem_u32(&full_bar[s]);
            const uint32_t bytes = kABytes + kBBytes + (has_sfa ? nvalid * 512 : 0) + w_tiles * nvalid * 512;
            mbar_arrive_expect_tx(fb, bytes);
            tma_load_2d(smem_u32(st), &map_a, fb, (int32_t)(ks * kBKBytes), (int32_t)(mt * kBM + rank * 128));
            tma_load_2d(smem_u32(st + kABytes), &map_w, fb, (int32_t)(ks * kBKBytes),
                        (int32_t)(n0 + rank * kBNHalf));
            if (has_sfa)
              bulk_load(smem_u32(st + kABytes + kBBytes), p.sfa + a_rt * p.sf_row_tile_bytes + g0 * 512,
                        nvalid * 512, fb);
            for (int t = 0; t < w_tiles; ++t)
              bulk_load(smem_u32(st + kABytes + kBBytes + kSfaBytes + t * 2048),
                        p.sfw + (w_rt + t) * p.sf_row_tile_bytes + g0 * 512, nvalid * 512, fb);
          }
        }
        if (!ok) {
          set_status(p.status, kStatusTimeout);
          *abort_flag = 1;
        }
        const uint32_t n_issued = it;
        for (uint32_t j = (n_issued > (uint32_t)kStages ? n_issued - kStages : 0); j < n_issued; ++j)
          mbar_wait_drain(smem_u32(&full_bar[j % kStages]), (j / kStages) & 1u, limit);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer (leader CTA)
      if (leader && lane == 0) {
        uint32_t it = 0, tcount = 0;
        bool ok = true;
        for (int64_t tile = pair; tile < p.num_tiles && ok; tile += num_pairs, ++tcount) {
          const int a = tcount % kAccStages;
          const uint32_t aph = (tcount / kAccStages) & 1u;
          if (!mbar_wait(smem_u32(&tempty_bar[a]), aph ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t d_tmem = tmem_base + a * kBN;
          for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&sf_bar[s]), ph, abort_flag, limit)) {
              ok = false;
              break;
            }
            fence_after();
            const int nvalid = (int)min((int64_t)4, p.num_k64 - ks * 4);
            uint8_t* st = smem + s * kStageBytes;
            const uint32_t a_addr = smem_u32(st), b_addr = smem_u32(st + kABytes);
            const uint32_t sf_slot = tmem_base + kSfColBase + s * kSfSlotCols;
            // descriptors of MMA k: start address + 32 k bytes, i.e. + 2 k in the
            // 16-byte address field (stage addresses stay far below its 2^18 bytes)
            const uint64_t ad0 = smem_desc(a_addr, 16, 1024, 2), bd0 = smem_desc(b_addr, 16, 1024, 2);
            if (nvalid == 4) {
  #pragma unroll
              for (int k = 0; k < 4; ++k)
                mma2(d_tmem, ad0 + 2 * k, bd0 + 2 * k, sf_slot + k * kSfPerMma, sf_slot + k * kSfPerMma + 4,
                     (ks > 0 || k > 0) ? 1u : 0u);
            } else {
              for (int k = 0; k < nvalid; ++k)
                mma2(d_tmem, ad0 + 2 * k, bd0 + 2 * k, sf_slot + k * kSfPerMma, sf_slot + k * kSfPerMma + 4,
                     (ks > 0 || k > 0) ? 1u : 0u);
            }
            commit2(smem_u32(&empty_bar[s]), (uint16_t)0x3);
          }
          if (!ok) break;
          commit2(smem_u32(&tfull_bar[a]), (uint16_t)0x3);
        }
        if (!ok) {
          set_status(p.status, kStatusTimeout);
          *abort_flag = 1;
        }
        commit2(smem_u32(done_bar), (uint16_t)0x1);
        mbar_wait_drain(smem_u32(done_bar), 0, limit);
      }
    }
  } else if (warp < kEpiWarp0) {
    regs_dec<kRegsSf>();
    // ------------------------------------------------------------ scale factors (both CTAs)
    // Slot of stage s, MMA k (c = kSfPerMma k): columns c + 0..3 hold this CTA's A
    // scales (lane l, column j: rows l + 32 j of its 128 rows), c + 4 .. c + 4 +
    // 4 kWTiles - 1 the W scales of all kBN rows of the pair tile (lane l, column j:
    // row l + 32 j).  Every group of 4 columns is line l of one of the stage's
    // 512-byte scale atoms.  The slot is rewritten only after the stage's TMA landed
    // again, i.e. after the MMAs that read it completed.
    const int quarter = warp & 3;
    const uint32_t leader_sf_bar0 = map_to_rank(smem_u32(&sf_bar[0]), 0);
    uint32_t it = 0;
    bool ok = true;
    for (int64_t tile = pair; tile < p.num_tiles && ok; tile += num_pairs) {
      const int64_t mt = tile % p.num_m, nt = tile / p.num_m;
      const bool has_sfa = mt * 2 + rank < p.a_row_tiles;
      const int64_t w_rt = nt * kBN / 128;
      for (int64_t ks = 0; ks < kstages; ++ks, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full_bar[s]), ph, abort_flag, limit))) {
          ok = false;
          break;
        }
        const int nvalid = (int)min((int64_t)4, p.num_k64 - ks * 4);
        const uint8_t* sfa = smem + s * kStageBytes + kABytes + kBBytes;
        const uint8_t* sfb = sfa + kSfaBytes;
        const uint32_t slot = tmem_base + ((uint32_t)(quarter * 32) << 16) + kSfColBase + s * kSfSlotCols;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 a = make_uint4(0, 0, 0, 0);
          if (k < nvalid && has_sfa) a = *reinterpret_cast<const uint4*>(sfa + k * 512 + lane * 16);
          tmem_st_32x32b_x4(slot + kSfPerMma * k, a);
#pragma unroll
          for (int t = 0; t < kWTiles; ++t) {
            uint4 b = make_uint4(0, 0, 0, 0);
            if (k < nvalid && w_rt + t < p.w_row_tiles)
              b = *reinterpret_cast<const uint4*>(sfb + t * 2048 + k * 512 + lane * 16);
            tmem_st_32x32b_x4(slot + kSfPerMma * k + 4 + 4 * t, b);
          }
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(leader_sf_bar0 + (uint32_t)(s * 8));
      }
    }
    if (!ok) {
      if (lane == 0) set_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
  } else {
    regs_inc<kRegsEpi>();
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Warp w reads tensor-memory lane quarter w % 4 (rows 32 (w % 4) .. + 31 of this
    // CTA's 128) and columns [64 g, 64 g + 64), g = (w - kEpiWarp0) / 4.  It takes
    // its 64 accumulator values into registers and frees the accumulator at once;
    // the scaling, activation, requantization and stores then overlap the next
    // tile's MMAs.
    const int quarter = warp & 3;
    const int cgroup = (warp - kEpiWarp0) / 4;
    const uint32_t leader_tempty0 = map_to_rank(smem_u32(&tempty_bar[0]), 0);
    const float gab = (*p.ga) * (*p.gw);
    const uint32_t buf = smem_u32(staging) + (uint32_t)((warp - kEpiWarp0) * kStagingBytesPerWarp);
    float gq = 0.0f, d6q = 0.0f, r6q = 0.0f;
    if (kFused && p.q_codes) {
      gq = *p.q_gscale_in;
      d6q = 6.0f * gq;
      r6q = 1.0f / d6q;
      if (blockIdx.x == 0 && threadIdx.x == kEpiWarp0 * 32) *p.q_gscale_out = gq;
    }
    const bool has_c = kFused ? p.has_c : true;
    // FP32 output goes through one 128-row box per column group; the group's 4 warps
    // synchronise on named barrier 1 + cgroup and so must also leave the tile loop
    // together.
    const bool grouped = has_c && !p.c_bf16;
    const uint32_t gbar = 1u + (uint32_t)cgroup;
    const uint32_t gbuf = smem_u32(staging) + (uint32_t)(cgroup * 4 * kStagingBytesPerWarp);
    unsigned amax_bits = 0;
    uint32_t tcount = 0;
    for (int64_t tile = pair; tile < p.num_tiles; tile += num_pairs, ++tcount) {
      const int a = tcount % kAccStages;
      const uint32_t aph = (tcount / kAccStages) & 1u;
      bool got = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&tfull_bar[a]), aph, abort_flag, limit));
      if (grouped) got = group_all(gbar, got);
      if (!got) {
        if (lane == 0) set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      fence_after();
      uint32_t r[2][32];
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + a * kBN + cgroup * 64;
      tmem_ld_32x32b_x32(taddr, r[0]);
      tmem_ld_32x32b_x32(taddr + 32, r[1]);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_tempty0 + (uint32_t)(a * 8));
      const int64_t mt = tile % p.num_m, nt = tile / p.num_m;
      const int32_t out_row = (int32_t)(mt * kBM + rank * 128 + quarter * 32);
      const int64_t row = (int64_t)out_row + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t col0 = nt * kBN + cgroup * 64 + h * 32;
        if (col0 >= p.N) break;  // warp-uniform
        float* v = reinterpret_cast<float*>(r[h]);
#pragma unroll
        for (int i = 0; i < 32; i += 2)
          mul2(v[i], v[i + 1], __uint_as_float(r[h][i]), __uint_as_float(r[h][i + 1]), gab, gab);
        if (kFused && p.act == 1) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) gelu_tanh2(v[i], v[i + 1]);
        }
        if (has_c) {
          if (p.c_bf16) {
            // the staging box is free once the previous store has read it
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 4; ++u)
              st_shared_v4(buf + lane * 64 + ((u ^ ((lane >> 1) & 3)) * 16),
                           make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                      pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7])));
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&map_c, buf, (int32_t)col0, out_row);
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
          } else {
            // FP32: the group's 4 warps fill one 128 x 16 box (8 KB), one thread stores it
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              if (quarter == 0 && lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
              asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory");
              const int rr = quarter * 32 + lane;
#pragma unroll
              for (int u = 0; u < 4; ++u)
                st_shared_v4(gbuf + rr * 64 + ((u ^ ((rr >> 1) & 3)) * 16),
                             make_uint4(__float_as_uint(v[16 * b + 4 * u]), __float_as_uint(v[16 * b + 4 * u + 1]),
                                        __float_as_uint(v[16 * b + 4 * u + 2]), __float_as_uint(v[16 * b + 4 * u + 3])));
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory");
              if (quarter == 0 && lane == 0) {
                tma_store_2d(&map_c, gbuf, (int32_t)(col0 + 16 * b), (int32_t)(mt * kBM + rank * 128));
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              }
            }
          }
        }
        if (!kFused) continue;
        if (row >= p.M) {
          // zero the scale padding of rows beyond M so the next GEMM reads finite scales
          if (p.q_codes && row < (p.M + 127) / 128 * 128)
            *reinterpret_cast<uint16_t*>(p.q_scales + sf_mma_offset(row, col0 / 16, p.q_groups)) = 0;
          continue;
        }
        const int nvc = (int)min((int64_t)32, p.N - col0);  // 16 on a ragged last chunk
        if (p.h_out) {
          float* hd = p.h_out + row * p.N + col0;
          if (nvc == 32) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              stg_v4(hd + 4 * q, make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                            __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3])));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nvc) hd[i] = v[i];
          }
        }
        if (p.q_amax_out && !p.q_codes) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nvc) amax_bits = max(amax_bits, __float_as_uint(v[i]) & 0x7FFFFFFFu);
        }
        if (p.q_codes) {  // N % 64 == 0 here, so the chunk is whole
          uint32_t w[4];
          uint32_t sc[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float s0[8], s1[8];
            // block max of |h|, NaN-propagating: a NaN makes the block's scale the
            // E4M3 NaN and (above +inf as bits) max|h| for q_amax_out non-finite
            float amax_b = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax_b = fmax_nan(amax_b, fabsf(v[16 * b + k]));
            amax_bits = max(amax_bits, __float_as_uint(amax_b));
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              s0[k] = v[16 * b + k];
              s1[k] = v[16 * b + 8 + k];
            }
            const uint32_t s = block_scale_fast(amax_b, d6q, r6q);
            const BlockEncoder enc(e4m3_to_float(s) * gq);
            w[2 * b] = enc.encode8s(s0);
            w[2 * b + 1] = enc.encode8s(s1);
            sc[b] = s;
          }
          stg_v4(p.q_codes + row * p.q_ld_codes + col0 / 2, make_uint4(w[0], w[1], w[2], w[3]));
          *reinterpret_cast<uint16_t*>(p.q_scales + sf_mma_offset(row, col0 / 16, p.q_groups)) =
              (uint16_t)(sc[0] | (sc[1] << 8));
        }
      }
    }
    if (kFused && p.q_amax_out) {
      amax_bits = warp_max_u32(amax_bits);
      if (lane == 0 && amax_bits) atomicMax(reinterpret_cast<unsigned*>(p.q_amax_out), amax_bits);
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  fence_before();
  cluster_sync();  // no CTA leaves while its peer may still use its shared or tensor memory
  fence_after();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
}

}  // namespace pair

// ----------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_relaxed);
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
      cached.store(fn, std::memory_order_relaxed);
    }
  }
  return fn;
}

// 2-D map over packed codes: inner dimension K/2 bytes, outer `rows`; box of
// 128 bytes x box_rows with the 128-byte swizzle the MMA descriptors assume.
bool make_code_map(CUtensorMap* m, const uint8_t* base, int64_t rows, int64_t kbytes, int64_t ld,
                   uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {(cuuint32_t)kBKBytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over the output C [M, N] (row pitch ldc elements) for the epilogue's
// TMA stores, boxes of `box_rows` rows swizzled like the staging buffers: 32
// columns (128 B rows, 128-byte swizzle, FP32; 64 B rows, 64-byte swizzle, bf16),
// or with `rows64` 64-byte rows for both types (16 FP32 or 32 bf16 columns).
bool make_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld, bool bf16,
                  bool rows64 = false, uint32_t box_rows = 32) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const int64_t esz = bf16 ? 2 : 4;
  const bool sw64 = bf16 || rows64;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * esz)};
  cuuint32_t box[2] = {(cuuint32_t)(sw64 ? 64 / esz : 32), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Opt a kernel into its dynamic shared memory once per device.
template <typename Kernel>
cudaError_t set_smem_once(Kernel k, int bytes, std::atomic<bool> (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!done[dev].load(std::memory_order_relaxed)) {  // setting it twice is harmless
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev].store(true, std::memory_order_relaxed);
  }
  return cudaSuccess;
}

int sm_count_gemm() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <bool kFused>
cudaError_t launch_gemm_pair(const GemmArgs& g, cudaStream_t s) {
  pair::Params2 p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.num_m = (g.M + pair::kBM - 1) / pair::kBM;
  p.num_n = (g.N + pair::kBN - 1) / pair::kBN;
  p.num_k64 = (g.K + kKPerMma - 1) / kKPerMma;
  p.num_tiles = p.num_m * p.num_n;
  p.a_row_tiles = (g.M + 127) / 128;
  p.w_row_tiles = (g.N + 127) / 128;
  p.sf_row_tile_bytes = p.num_k64 * 512;
  p.sfa = g.a.scales;
  p.sfw = g.w.scales;
  p.ga = g.a.gscale;
  p.gw = g.w.gscale;
  p.has_c = g.c != nullptr;
  p.c_bf16 = g.c_bf16;
  p.act = g.act;
  p.q_codes = g.q_codes;
  p.q_ld_codes = g.q_ld_codes;
  p.q_scales = g.q_scales;
  p.q_groups = (g.N / 16 + 3) / 4;
  p.q_gscale_in = g.q_gscale_in;
  p.q_gscale_out = g.q_gscale_out;
  p.q_amax_out = g.q_amax_out;
  p.h_out = g.h_out;
  p.status = g.status;
  p.wait_limit_ns = g_debug_wait_limit_ns.load() ? g_debug_wait_limit_ns.load() : kWaitLimitNs;
  p.drop_first_stage = g_debug_drop_first_stage.load();

  CUtensorMap ma, mw, mc;
  if (!make_code_map(&ma, g.a.codes, g.M, g.K / 2, g.a.ld_codes, 128)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, g.w.codes, g.N, g.K / 2, g.w.ld_codes, pair::kBNHalf)) return cudaErrorInvalidValue;
  memset(&mc, 0, sizeof(mc));
  // FP32 output: one 128-row box per column group of the epilogue (see the kernel)
  if (g.c && !make_out_map(&mc, g.c, g.M, g.N, g.ldc, g.c_bf16, true, g.c_bf16 ? 32u : 128u))
    return cudaErrorInvalidValue;
  if (g.q_amax_out) {
    cudaError_t e = launch_zero_words(g.q_amax_out, 1, s);
    if (e != cudaSuccess) return e;
  }
  static std::atomic<bool> done[64];
  cudaError_t e = set_smem_once(pair::gemm_pair_kernel<kFused>, pair::kSmemBytes, done);
  if (e != cudaSuccess) return e;
  // Pairs must fit inside one GPC, so fewer than SMs / 2 of them may be resident
  // at once; a persistent grid larger than that would run a second wave.
  static std::atomic<int> resident[64];
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (resident[dev].load(std::memory_order_relaxed) == 0) {
    // The kernel's register split (setmaxnreg) balances only for this launch count:
    // with fewer registers at launch its epilogue warps would wait for registers
    // that are never released.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, pair::gemm_pair_kernel<kFused>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != pair::kRegsLaunch) return cudaErrorInvalidKernelImage;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * (sm_count_gemm() / 2)), 1, 1);
    cfg.blockDim = dim3(pair::kThreads, 1, 1);
    cfg.dynamicSmemBytes = pair::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, pair::gemm_pair_kernel<kFused>, &cfg);
    if (e != cudaSuccess) return e;
    if (n <= 0) return cudaErrorInvalidConfiguration;
    resident[dev].store(n, std::memory_order_relaxed);
  }
  const int64_t max_pairs = resident[dev].load(std::memory_order_relaxed);
  const int64_t pairs = p.num_tiles < max_pairs ? p.num_tiles : max_pairs;
  launch_pdl(pair::gemm_pair_kernel<kFused>, (unsigned)(2 * pairs), pair::kThreads, pair::kSmemBytes, s, ma, mw, mc, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
  if (g.M == 0 || g.N == 0) return cudaSuccess;
  // At least one full pair tile of rows and columns: the CTA-pair kernel (256 x 256
  // tiles), its plain-output instance or the one with the general epilogue.  Smaller
  // shapes: the single-CTA kernel (128 x 128 tiles).
  const bool plain = g.c != nullptr && g.act == 0 && g.q_codes == nullptr && g.h_out == nullptr &&
                     g.q_amax_out == nullptr;
  if (g.M >= pair::kBM && g.N >= pair::kBN)
    return plain ? launch_gemm_pair<false>(g, s) : launch_gemm_pair<true>(g, s);
  Params p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.num_m = (g.M + kBM - 1) / kBM;
  p.num_n = (g.N + kBN - 1) / kBN;
  p.num_k64 = (g.K + kKPerMma - 1) / kKPerMma;
  p.num_tiles = p.num_m * p.num_n;
  p.sfa_row_tile_bytes = p.num_k64 * 512;
  p.sfw_row_tile_bytes = p.num_k64 * 512;
  p.sfa = g.a.scales;
  p.sfw = g.w.scales;
  p.ga = g.a.gscale;
  p.gw = g.w.gscale;
  p.c = (uint8_t*)g.c;
  p.c_bf16 = g.c_bf16;
  p.ldc = g.ldc;
  p.act = g.act;
  p.q_codes = g.q_codes;
  p.q_ld_codes = g.q_ld_codes;
  p.q_scales = g.q_scales;
  p.q_groups = (g.N / 16 + 3) / 4;
  p.q_gscale_in = g.q_gscale_in;
  p.q_gscale_out = g.q_gscale_out;
  p.q_amax_out = g.q_amax_out;
  p.h_out = g.h_out;
  p.status = g.status;
  p.wait_limit_ns = g_debug_wait_limit_ns.load() ? g_debug_wait_limit_ns.load() : kWaitLimitNs;
  p.drop_first_stage = g_debug_drop_first_stage.load();

  CUtensorMap ma, mw;
  if (!make_code_map(&ma, g.a.codes, g.M, g.K / 2, g.a.ld_codes, kBM)) return cudaErrorInvalidValue;
  if (!make_code_map(&mw, g.w.codes, g.N, g.K / 2, g.w.ld_codes, kBN)) return cudaErrorInvalidValue;
  CUtensorMap mc;
  memset(&mc, 0, sizeof(mc));
  if (g.c && !make_out_map(&mc, g.c, g.M, g.N, g.ldc, g.c_bf16)) return cudaErrorInvalidValue;

  if (g.q_amax_out) {
    cudaError_t e = launch_zero_words(g.q_amax_out, 1, s);
    if (e != cudaSuccess) return e;
  }
  static std::atomic<bool> done[64];
  cudaError_t e = set_smem_once(gemm_kernel, kSmemBytes, done);
  if (e != cudaSuccess) return e;
  const int sms = sm_count_gemm();
  const int grid = (int)(p.num_tiles < sms ? p.num_tiles : sms);
  launch_pdl(gemm_kernel, grid, kThreads, kSmemBytes, s, ma, mw, mc, p);
  return cudaGetLastError();
}

void gemm_debug_fault(int drop_first_stage, unsigned long long wait_limit_ns) {
  g_debug_drop_first_stage.store(drop_first_stage ? 1 : 0);
  g_debug_wait_limit_ns.store(wait_limit_ns);
}

}  // namespace nvfp4
