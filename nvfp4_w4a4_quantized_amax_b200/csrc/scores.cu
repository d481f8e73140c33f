// scores.cu — attention scores and outputs straight from the NVFP4 KV cache.
//
// techwalker.com, "NVIDIA研究团队打造全球首个FP4视频生成系统，速度提升两倍还省一半内存", §四:
// K and V are kept in NVFP4 (K after subtracting its mean) and the chunks of the
// attention window are dequantized together.  Here the K side of that window is
// consumed by the attention product itself: each CTA dequantizes one tile of 128
// window keys of one head from the cache into shared memory (never to HBM), in the
// tensor core's 128-byte-swizzled K-major layout, and multiplies every query tile of
// that head with it on the tcgen05 tensor cores (kind::f16, bf16 x bf16, FP32
// accumulators in tensor memory):
//
//   S[h, i, j] = RN(scale * sum_d Q[i, h, d] * K^[j, h, d])     (FP32 accumulate)
//   K^[j, h, d] = bf16(RN(RN(e2m1 * s * g_K) + mu[h, d]))      (the window's K, bit for
//                                                               bit what kv_dequant_window
//                                                               writes)
//
// A persistent kernel (one CTA per SM) walks the (key tile, head) items; while one
// item's query tiles go through the tensor cores and the epilogue, six warps decode
// the next item's keys into a second buffer.  The dequantized keys are reused by every
// query tile, so the cache is read once per (head, key tile) and no bf16 copy of the
// window exists in HBM.  The V side (P V^) follows below.
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nvfp4 {
namespace {

using namespace tc;

constexpr int kQ = 128;          // queries per tile (MMA M, tensor-memory lanes)
constexpr int kKeys = 128;       // keys per work item (MMA N)
constexpr int kD = 128;          // head_dim (MMA K, 8 instructions of 16)
constexpr int kThreads = 512;    // 16 warps
constexpr int kQBufs = 3;
constexpr int kKBufs = 2;
constexpr int kAcc = 4;
constexpr int kEpiWarp0 = 4, kEpiWarps = 8;
constexpr int kDecThreads = 192;  // warps 2, 3 and 12..15
constexpr int kKBytes = kKeys * kD * 2;  // 32 KB: two 128-row x 128-byte swizzled blocks
constexpr int kQBytes = kQ * kD * 2;     // 32 KB
constexpr int kBlockBytes = 128 * 128;   // one 64-column block of a 128-row tile
constexpr int kBoxBytes = 32 * 128;      // one output box: 32 query rows x 128 bytes
constexpr int kStageBytes = kEpiWarps * 2 * kBoxBytes;  // two boxes in flight per epilogue warp
constexpr int kSmemBytes =
    kKBufs * kKBytes + kQBufs * kQBytes + kStageBytes + 1024 /*barriers*/ + 1024 /*alignment*/;
constexpr int kDecRowStep = kDecThreads / 16;  // 12: a thread's rows are r0, r0 + 12, ...
constexpr int kRowsPerDecThread = (kKeys + kDecRowStep - 1) / kDecRowStep;  // at most 11
constexpr int kTmemCols = kAcc * kKeys;  // 512
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// kind::f16: D FP32 (bits 4..5 = 1), A and B bf16 (bits 7..9, 10..12 = 1), both
// K-major, N >> 3 at bits 17..22, M >> 4 at bits 24..28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKeys >> 3) << 17) |
                            ((uint32_t)(kQ >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

struct ScoresParams {
  const uint8_t* base;
  int64_t off_k_codes, off_k_scales, off_mu, off_gscale, off_tokens;
  int64_t slot_codes_bytes, slot_scales_bytes;
  int32_t heads, n_slots;
  int32_t slots[kMaxWindowSlots];
  int32_t tokens[kMaxWindowSlots];
  int64_t key_end[kMaxWindowSlots];  // cumulative window keys through list entry i
  int64_t Tq, Tk;
  int64_t n_items;                   // key tiles x heads
  float scale;
  bool s_bf16;
  unsigned* status;
  unsigned long long wait_limit_ns;
};

// CTA: a persistent loop over work items (key tile kt, head h), items c, c + grid, ...
// of the n_kt * heads in head-major order; one CTA per SM.  16 warps:
//   warp 0      TMA producer: every query tile of every item in turn (128 queries x
//               128 dims bf16, two 64-column boxes, 128-byte swizzle), kQBufs buffers
//   warp 1      MMA issuer: 8 tcgen05.mma (K = 16 each) per query tile into one of kAcc
//               128-column accumulators; an item's K^ buffer is released after its
//               last query tile
//   warps 4..11 epilogue: warp w takes tensor-memory lane quarter w % 4 and the 64 keys
//               [64 (w - 4) / 4, ..) of the tile: tcgen05.ld of a query row's scores,
//               scaling, 32-row x 128-byte boxes staged in shared memory (128-byte
//               swizzle) and written by TMA stores clipped to the head's queries and the
//               window's keys
//   warps 2, 3, 12..15 dequantize the next item's 128 keys x 128 dims straight from
//               the cache into the other of two K^ buffers (the MMA's 128-byte-swizzled
//               K-major layout) while the current item runs
// Each (head, key tile) of K is read from the cache once and no bf16 copy of the
// window exists in HBM.  Every wait is bounded (2 s): a wait that gives up records
// NVFP4_ERR_TIMEOUT, the CTA drains its own copies and MMAs and leaves.
__global__ void __launch_bounds__(kThreads, 1)
    kv_scores_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_s,
                     const __grid_constant__ ScoresParams p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kbuf = smem;                              // kKBufs K^ tiles, 1024-aligned
  uint8_t* qbuf = kbuf + kKBufs * kKBytes;           // kQBufs query tiles
  uint8_t* stage = qbuf + kQBufs * kQBytes;          // output boxes, 8 KB per epilogue warp
  uint8_t* bar_area = stage + kStageBytes;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* q_empty = q_full + kQBufs;
  uint64_t* k_full = q_empty + kQBufs;
  uint64_t* k_empty = k_full + kKBufs;
  uint64_t* t_full = k_empty + kKBufs;
  uint64_t* t_empty = t_full + kAcc;
  uint64_t* done_bar = t_empty + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* valid = reinterpret_cast<int32_t*>(tmem_slot + 2);         // per list entry: its slot holds the count
  float* gk_tab = reinterpret_cast<float*>(valid + kMaxWindowSlots);  // per list entry: g_K of its slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_kt = (p.Tk + kKeys - 1) / kKeys;
  const int64_t n_qt = (p.Tq + kQ - 1) / kQ;
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
  const uint32_t n_my = p.n_items > blockIdx.x ? (uint32_t)((p.n_items - 1 - blockIdx.x) / gridDim.x + 1) : 0u;
  const unsigned long long limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kQBufs; ++b) {
      mbar_init(smem_u32(&q_full[b]), 1);
      mbar_init(smem_u32(&q_empty[b]), 1);
    }
    for (int b = 0; b < kKBufs; ++b) {
      mbar_init(smem_u32(&k_full[b]), kDecThreads / 32);
      mbar_init(smem_u32(&k_empty[b]), 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(smem_u32(&t_full[a]), 1);
      mbar_init(smem_u32(&t_empty[a]), kEpiWarps);
    }
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
  pdl_wait();  // the cache, the queries and the output buffer come from earlier work
  if (threadIdx.x < p.n_slots) {
    const int i = threadIdx.x;
    const bool ok = reinterpret_cast<const int32_t*>(p.base + p.off_tokens)[p.slots[i]] == p.tokens[i];
    valid[i] = ok ? 1 : 0;
    gk_tab[i] = reinterpret_cast<const float*>(p.base + p.off_gscale)[2 * p.slots[i]];
    if (!ok && blockIdx.x == 0) set_status(p.status, kStatusShape);  // the slot holds another token count
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ query producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
      bool ok = true;
      uint32_t u = 0;  // query tiles issued, over all items
      for (uint32_t w = 0; w < n_my && ok; ++w) {
        const int h = (int)((blockIdx.x + (int64_t)w * gridDim.x) / n_kt);
        for (uint32_t qt = 0; qt < (uint32_t)n_qt; ++qt, ++u) {
          const int b = u % kQBufs;
          if (!mbar_wait(smem_u32(&q_empty[b]), ((u / kQBufs) & 1u) ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&q_full[b]);
          mbar_arrive_expect_tx(fb, kQBytes);
          uint8_t* dst = qbuf + b * kQBytes;
          tma_load_2d(smem_u32(dst), &map_q, fb, h * kD, (int32_t)(qt * kQ));
          tma_load_2d(smem_u32(dst + kBlockBytes), &map_q, fb, h * kD + 64, (int32_t)(qt * kQ));
        }
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      for (uint32_t j = u > (uint32_t)kQBufs ? u - kQBufs : 0; j < u; ++j)
        mbar_wait_drain(smem_u32(&q_full[j % kQBufs]), (j / kQBufs) & 1u, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      uint32_t u = 0;
      for (uint32_t w = 0; w < n_my && ok; ++w) {
        const int kb = w % kKBufs;
        if (!mbar_wait(smem_u32(&k_full[kb]), (w / kKBufs) & 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        const uint32_t k_addr = smem_u32(kbuf + kb * kKBytes);
        for (uint32_t qt = 0; qt < (uint32_t)n_qt; ++qt, ++u) {
          const int b = u % kQBufs, a = u % kAcc;
          if (!mbar_wait(smem_u32(&t_empty[a]), ((u / kAcc) & 1u) ^ 1u, abort_flag, limit) ||
              !mbar_wait(smem_u32(&q_full[b]), (u / kQBufs) & 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t q_addr = smem_u32(qbuf + b * kQBytes);
          const uint32_t d_tmem = tmem_base + a * kKeys;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            // K = 16 bf16 = 32 bytes of each swizzled 128-byte row: 4 per 64-column block
            const uint32_t off = (kk >> 2) * kBlockBytes + (kk & 3) * 32;
            mma_bf16(d_tmem, smem_desc(q_addr + off, 16, 1024, 2), smem_desc(k_addr + off, 16, 1024, 2),
                     kk > 0 ? 1u : 0u);
          }
          commit(smem_u32(&q_empty[b]));
          commit(smem_u32(&t_full[a]));
        }
        if (ok) commit(smem_u32(&k_empty[kb]));
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      commit(smem_u32(done_bar));
      mbar_wait_drain(smem_u32(done_bar), 0, limit);
    }
  } else if (warp < kEpiWarp0 || warp >= kEpiWarp0 + kEpiWarps) {
    // ------------------------------------------------------------ K^ producers
    // thread t: the 8-dim chunk c16 = t % 16 of key rows t / 16 + 12 u below 128;
    // K^[j, h, d] = bf16(RN(RN(e2m1 * s * g_K) + mu[h, d])), zeros beyond the window
    const int t = (warp < kEpiWarp0 ? warp - 2 : warp - 10) * 32 + lane;
    const int c16 = t & 15, r0 = t >> 4;
    const int d0 = c16 * 8;
    const int blk = d0 >> 6, cch = (d0 & 63) >> 3;
    bool ok = true;
    for (uint32_t w = 0; w < n_my; ++w) {
      const int64_t item = blockIdx.x + (int64_t)w * gridDim.x;
      const int h = (int)(item / n_kt);
      const int64_t kt = item - (int64_t)h * n_kt;
      // every code word and scale byte of this thread's rows in flight at once
      uint32_t kcw[kRowsPerDecThread], ksb[kRowsPerDecThread];
      int32_t rseg[kRowsPerDecThread];
      int seg = 0;
#pragma unroll
      for (int u = 0; u < kRowsPerDecThread; ++u) {
        const int64_t j = kt * kKeys + r0 + kDecRowStep * u;
        kcw[u] = 0;
        ksb[u] = 0;
        rseg[u] = -1;
        if (r0 + kDecRowStep * u < kKeys && j < p.Tk) {
          while (j >= p.key_end[seg]) ++seg;
          if (valid[seg]) {
            const int slot = p.slots[seg];
            const int64_t e = ((j - (seg == 0 ? 0 : p.key_end[seg - 1])) * p.heads + h) * kD + d0;
            kcw[u] = __ldg(reinterpret_cast<const uint32_t*>(p.base + p.off_k_codes + slot * p.slot_codes_bytes + e / 2));
            ksb[u] = __ldg(p.base + p.off_k_scales + slot * p.slot_scales_bytes + e / 16);
            rseg[u] = seg;
          }
        }
      }
      const int kb = w % kKBufs;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&k_empty[kb]), ((w / kKBufs) & 1u) ^ 1u, abort_flag, limit))) {
        ok = false;
        break;
      }
      uint8_t* kdst = kbuf + kb * kKBytes + blk * kBlockBytes;
      int cur = -1;
      float gk = 0.0f;
      float mu[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mu[q] = 0.0f;
#pragma unroll
      for (int u = 0; u < kRowsPerDecThread; ++u) {
        const int r = r0 + kDecRowStep * u;
        if (r >= kKeys) break;
        uint4 out = make_uint4(0, 0, 0, 0);
        if (rseg[u] >= 0) {
          if (rseg[u] != cur) {  // g_K and this chunk's mu of the row's slot
            cur = rseg[u];
            const int slot = p.slots[cur];
            gk = gk_tab[cur];
            const float4* m4 = reinterpret_cast<const float4*>(
                p.base + p.off_mu + (((int64_t)slot * p.heads + h) * kD + d0) * 4);
            const float4 m0 = __ldg(m4), m1 = __ldg(m4 + 1);
            mu[0] = m0.x; mu[1] = m0.y; mu[2] = m0.z; mu[3] = m0.w;
            mu[4] = m1.x; mu[5] = m1.y; mu[6] = m1.z; mu[7] = m1.w;
          }
          uint32_t kh[4];
          e2m1x8_times_scale(kcw[u], e4m3_to_f16x2_bcast(ksb[u]), kh);
          float ko[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) f16x2_to_f32x2(kh[q], ko[2 * q], ko[2 * q + 1]);  // e2m1 * s, exact
#pragma unroll
          for (int q = 0; q < 8; ++q)  // two roundings: the product, then the sum
            ko[q] = __fadd_rn(__fmul_rn(ko[q], gk), mu[q]);
          out = make_uint4(pack_bf16x2(ko[0], ko[1]), pack_bf16x2(ko[2], ko[3]), pack_bf16x2(ko[4], ko[5]),
                           pack_bf16x2(ko[6], ko[7]));
        }
        // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
        *reinterpret_cast<uint4*>(kdst + r * 128 + ((cch ^ (r & 7)) << 4)) = out;
      }
      fence_proxy_async_smem();  // the tensor core reads K^ through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&k_full[kb]));
    }
    if (!ok) {
      if (lane == 0) set_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - kEpiWarp0) >> 2;  // keys [64 half, 64 half + 64) of the tile
    const int cols = p.s_bf16 ? 64 : 32;       // keys per box
    const uint32_t wbuf = smem_u32(stage) + (uint32_t)((warp - kEpiWarp0) * 2 * kBoxBytes);
    uint32_t nbox = 0, u = 0;
    bool ok = true;
    for (uint32_t w = 0; w < n_my && ok; ++w) {
      const int64_t item = blockIdx.x + (int64_t)w * gridDim.x;
      const int h = (int)(item / n_kt);
      const int64_t key0 = (item - (int64_t)h * n_kt) * kKeys + 64 * half;
      for (uint32_t qt = 0; qt < (uint32_t)n_qt; ++qt, ++u) {
        const int a = u % kAcc;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&t_full[a]), (u / kAcc) & 1u, abort_flag, limit))) {
          ok = false;
          break;
        }
        fence_after();
        const uint32_t trow = tmem_base + ((uint32_t)(quarter * 32) << 16) + a * kKeys + 64 * half;
#pragma unroll 1
        for (int c0 = 0; c0 < 64 && key0 + c0 < p.Tk; c0 += cols, ++nbox) {  // warp-uniform
          uint32_t wv[32];  // the row's 128 bytes of this box
          {
            uint32_t r[32];
            tmem_ld_32x32b_x32(trow + c0, r);
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              mul2(v[i], v[i + 1], __uint_as_float(r[i]), __uint_as_float(r[i + 1]), p.scale, p.scale);
            if (p.s_bf16) {
#pragma unroll
              for (int i = 0; i < 16; ++i) wv[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
              tmem_ld_32x32b_x32(trow + c0 + 32, r);
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                mul2(v[i], v[i + 1], __uint_as_float(r[i]), __uint_as_float(r[i + 1]), p.scale, p.scale);
#pragma unroll
              for (int i = 0; i < 16; ++i) wv[16 + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) wv[i] = __float_as_uint(v[i]);
            }
          }
          const uint32_t buf = wbuf + (nbox & 1u) * kBoxBytes;
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)  // 128-byte swizzle: chunk c of row r at chunk c ^ (r % 8)
            st_shared_v4(buf + lane * 128 + ((c ^ (lane & 7)) << 4),
                         make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&map_s, buf, (int32_t)(key0 + c0), (int32_t)(qt * kQ + quarter * 32), h);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&t_empty[a]));
      }
    }
    if (!ok) {
      if (lane == 0) set_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete
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

// ============================================================ the V side
// O[i, h, d] = sum_j P[h, i, j] * V^[j, h, d] over the window's keys j, with
//   V^[j, h, d] = bf16(RN(RN(e2m1 * s) * g_V))   (the window's V, bit for bit)
// and P given (e.g. the softmax of the scores), FP32 accumulation in tensor memory.
// A CTA takes G <= 4 query tiles of 128 queries of one head (G accumulators of 128
// columns in tensor memory), so each 64-key tile of V^ it dequantizes feeds G tiles of
// P; a cluster of S CTAs splits the window's key tiles into S contiguous ranges.  The
// host picks G and S for the fewest waves of the longest CTA.  12 warps:
//   warp 0      TMA producer: per key tile, G boxes of P (128 queries x 64 keys bf16,
//               128-byte swizzle) into a ring of kPSlots 16 KB slots
//   warp 1      MMA issuer: per key tile and query tile, 4 tcgen05.mma (K = 16 keys),
//               each P slot released as soon as its MMAs complete
//   warps 4..11 dequantize each key tile's V^ into shared memory transposed (128 dims
//               x 64 keys: the MMA's K-major B operand), two buffers.  The cache's code
//               words, scale bytes and g_V of a key tile are staged with cp.async
//               (coalesced: four threads per key) in a ring of kRing tiles, kRing - 1
//               tiles ahead of the decode.  Warps 4..7 (one lane quarter each) then read
//               the accumulators.
// With S = 1 the accumulators go straight to the output.  With S > 1, query tile by
// query tile, every CTA puts its partial in shared memory and CTA r sums rows
// [128 r / S, 128 (r + 1) / S) over the cluster in rank order (distributed shared
// memory; a fixed order, so the result does not depend on scheduling).
constexpr int kCtxThreads = 384;
constexpr int kCtxKeys = 64;                          // keys per tile (K of 4 MMAs)
constexpr int kCtxMaxG = 4;                           // query tiles per CTA
constexpr int kPTileBytes = kQ * kCtxKeys * 2;        // 16 KB: 128 queries x 64 keys
constexpr int kPSlots = 10;                           // P tiles in flight
constexpr int kVTBytes = kD * kCtxKeys * 2;           // 16 KB: 128 dims x 64 keys
constexpr int kCtxVBufs = 2;
constexpr int kVWarp0 = 4;
constexpr int kVThreads = 256;                        // warps 4..11
constexpr int kRing = 5;                              // key tiles of V cache data in flight
// one staged key tile: code bytes [8 dim groups of 16][64 keys] x 8 B, scale bytes
// [64 keys] x 8 B (one per dim group), g_V [64 keys] x 4 B
constexpr int kRingCodes = 8 * kCtxKeys * 8;
constexpr int kRingScales = kRingCodes;
constexpr int kRingGv = kRingScales + kCtxKeys * 8;
constexpr int kRingStageBytes = kRingGv + kCtxKeys * 4 + 256;  // 5 KB
constexpr int kPartRowBytes = kD * 4;                 // one query row of an FP32 partial
constexpr int kCtxSmemBytes = kPSlots * kPTileBytes + kCtxVBufs * kVTBytes + kRing * kRingStageBytes +
                              1024 /*barriers*/ + 1024 /*alignment*/;
static_assert(kPSlots * kPTileBytes >= kQ * kPartRowBytes, "a partial tile reuses the P slots");
constexpr int kCtxTmemCols = kCtxMaxG * kD;           // 512
constexpr int kMaxSplit = 8;

struct ContextParams {
  const uint8_t* base;
  int64_t off_v_codes, off_v_scales, off_gscale, off_tokens;
  int64_t slot_codes_bytes, slot_scales_bytes;
  int32_t heads, n_slots;
  int32_t slots[kMaxWindowSlots];
  int32_t tokens[kMaxWindowSlots];
  int64_t key_end[kMaxWindowSlots];
  int64_t Tq, Tk;
  int64_t tiles_per_split;  // key tiles per CTA of a cluster
  int32_t split;            // S: CTAs per (query group, head) = cluster size
  int32_t G;                // query tiles per CTA
  int32_t n_qt;             // query tiles in all
  bool o_bf16;
  uint8_t* o;
  int64_t ldo;
  unsigned* status;
  unsigned long long wait_limit_ns;
};

// Where key j of the window lies in the cache: the byte offsets of its 64 code bytes
// and 8 scale bytes for head h, and its list entry (seg); false beyond the window or
// for a slot that holds another token count.
__device__ __forceinline__ bool ctx_locate(const ContextParams& p, const int32_t* valid, int64_t j, int h, int& seg,
                                           int64_t& codes_off, int64_t& scales_off) {
  if (j >= p.Tk) return false;
  while (j >= p.key_end[seg]) ++seg;  // keys only grow along a CTA's range
  if (!valid[seg]) return false;
  const int slot = p.slots[seg];
  const int64_t th = (j - (seg == 0 ? 0 : p.key_end[seg - 1])) * p.heads + h;  // (token, head) within the slot
  codes_off = p.off_v_codes + slot * p.slot_codes_bytes + th * (kD / 2);
  scales_off = p.off_v_scales + slot * p.slot_scales_bytes + th * (kD / 16);
  return true;
}

// 16 dims of one key as floats: e2m1 * s exactly (f16), then one FP32 product with g_V.
__device__ __forceinline__ void ctx_decode(uint32_t w0, uint32_t w1, uint32_t sbyte, float gv, float (&f)[16]) {
  const uint32_t s2 = e4m3_to_f16x2_bcast(sbyte);
  uint32_t h0[4], h1[4];
  e2m1x8_times_scale(w0, s2, h0);  // dims 0..7
  e2m1x8_times_scale(w1, s2, h1);  // dims 8..15
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float lo, hi;
    f16x2_to_f32x2(h0[q], lo, hi);  // e2m1 * s, exact
    mul2(f[2 * q], f[2 * q + 1], lo, hi, gv, gv);
    f16x2_to_f32x2(h1[q], lo, hi);
    mul2(f[8 + 2 * q], f[9 + 2 * q], lo, hi, gv, gv);
  }
}

// bar.red.or over the `count` threads of named barrier `id`: true if any passed true.
__device__ __forceinline__ bool named_barrier_or(uint32_t id, uint32_t count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// kind::f16 again (M = N = 128); the B operand is V^ transposed (dims x keys).
__global__ void __launch_bounds__(kCtxThreads, 1)
    kv_context_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ ContextParams p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* pbuf = smem;                                // P slots; the partial output at the end
  uint8_t* vbuf = smem + kPSlots * kPTileBytes;        // V^T tiles
  uint8_t* ring = vbuf + kCtxVBufs * kVTBytes;         // V cache data in flight
  uint8_t* bar_area = ring + kRing * kRingStageBytes;
  uint64_t* p_full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* p_empty = p_full + kPSlots;
  uint64_t* v_full = p_empty + kPSlots;
  uint64_t* v_empty = v_full + kCtxVBufs;
  uint64_t* t_full = v_empty + kCtxVBufs;
  uint64_t* done_bar = t_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* valid = reinterpret_cast<int32_t*>(tmem_slot + 2);         // per list entry: its slot holds the count
  float* gv_tab = reinterpret_cast<float*>(valid + kMaxWindowSlots);  // per list entry: g_V of its slot
  volatile int* acc_ok = reinterpret_cast<volatile int*>(gv_tab + kMaxWindowSlots);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = blockIdx.x, qg = blockIdx.y, h = blockIdx.z;  // rank = this CTA's rank in its cluster
  const int qt0 = qg * p.G;
  const int G = p.n_qt - qt0 < p.G ? p.n_qt - qt0 : p.G;         // this CTA's query tiles
  const int64_t n_kt = (p.Tk + kCtxKeys - 1) / kCtxKeys;
  const int64_t kt0 = rank * p.tiles_per_split;
  const int64_t kt_end = kt0 + p.tiles_per_split < n_kt ? kt0 + p.tiles_per_split : n_kt;
  const uint32_t n_my = kt_end > kt0 ? (uint32_t)(kt_end - kt0) : 0u;
  const unsigned long long limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int b = 0; b < kPSlots; ++b) {
      mbar_init(smem_u32(&p_full[b]), 1);
      mbar_init(smem_u32(&p_empty[b]), 1);
    }
    for (int b = 0; b < kCtxVBufs; ++b) {
      mbar_init(smem_u32(&v_full[b]), kVThreads / 32);
      mbar_init(smem_u32(&v_empty[b]), 1);
    }
    mbar_init(smem_u32(t_full), 1);
    mbar_init(smem_u32(done_bar), 1);
    *abort_flag = 0;
    *acc_ok = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kCtxTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();  // the cache and P come from earlier work
  if (threadIdx.x < p.n_slots) {
    const int i = threadIdx.x;
    const bool ok = reinterpret_cast<const int32_t*>(p.base + p.off_tokens)[p.slots[i]] == p.tokens[i];
    valid[i] = ok ? 1 : 0;
    gv_tab[i] = reinterpret_cast<const float*>(p.base + p.off_gscale)[2 * p.slots[i] + 1];
    if (!ok && rank == 0) set_status(p.status, kStatusShape);  // the slot holds another token count
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ P producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_p)) : "memory");
      bool ok = true;
      uint32_t c = 0;  // P tiles issued: tile g of key tile i is the (i G + g)-th
      for (uint32_t i = 0; i < n_my && ok; ++i) {
        const int32_t key = (int32_t)((kt0 + i) * kCtxKeys);
        for (int g = 0; g < G; ++g, ++c) {
          const uint32_t sl = c % kPSlots;
          if (!mbar_wait(smem_u32(&p_empty[sl]), ((c / kPSlots) & 1u) ^ 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&p_full[sl]);
          mbar_arrive_expect_tx(fb, (uint32_t)kPTileBytes);
          tma_load_3d(smem_u32(pbuf + sl * kPTileBytes), &map_p, fb, key, (qt0 + g) * kQ, h);
        }
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      for (uint32_t j = c > (uint32_t)kPSlots ? c - kPSlots : 0; j < c; ++j)
        mbar_wait_drain(smem_u32(&p_full[j % kPSlots]), (j / kPSlots) & 1u, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      uint32_t c = 0;  // P tiles consumed, in the producer's order
      for (uint32_t i = 0; i < n_my && ok; ++i) {
        const int bv = i % kCtxVBufs;
        if (!mbar_wait(smem_u32(&v_full[bv]), (i / kCtxVBufs) & 1u, abort_flag, limit)) {
          ok = false;
          break;
        }
        const uint32_t b_addr = smem_u32(vbuf + bv * kVTBytes);
        for (int g = 0; g < G; ++g, ++c) {
          const uint32_t sl = c % kPSlots;
          if (!mbar_wait(smem_u32(&p_full[sl]), (c / kPSlots) & 1u, abort_flag, limit)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t a_addr = smem_u32(pbuf + sl * kPTileBytes);
#pragma unroll
          for (int kk = 0; kk < kCtxKeys / 16; ++kk)
            mma_bf16(tmem_base + (uint32_t)(g * kD), smem_desc(a_addr + kk * 32, 16, 1024, 2),
                     smem_desc(b_addr + kk * 32, 16, 1024, 2), (i > 0 || kk > 0) ? 1u : 0u);
          commit(smem_u32(&p_empty[sl]));
        }
        if (ok) commit(smem_u32(&v_empty[bv]));
      }
      if (!ok) {
        set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      } else {
        commit(smem_u32(t_full));
      }
      commit(smem_u32(done_bar));
      mbar_wait_drain(smem_u32(done_bar), 0, limit);
    }
  } else if (warp >= kVWarp0) {
    // ------------------------------------------------------------ V^T producers
    const int t = threadIdx.x - kVWarp0 * 32;  // 0..255
    // staging (cp.async): key ck = t / 4 of the tile, its code bytes [16 cc, 16 cc + 16)
    // (dims [32 cc, 32 cc + 32), dim groups 2 cc and 2 cc + 1); threads t < 64 also
    // stage key t's 8 scale bytes and its g_V
    const int ck = t >> 2, cc = t & 3;
    int seg_c = 0, seg_s = 0;
    auto issue = [&](uint32_t i) {
      uint8_t* st = ring + (i % kRing) * kRingStageBytes;
      const int64_t j0 = (kt0 + i) * kCtxKeys;
      int64_t co = 0, so = 0;
      const bool okc = ctx_locate(p, valid, j0 + ck, h, seg_c, co, so);
      const uint8_t* src = p.base + (okc ? co + 16 * cc : 0);
      const uint32_t n = okc ? 8u : 0u;  // zero-filled beyond the window or for a stale slot
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(st + ((2 * cc) * kCtxKeys + ck) * 8)),
                   "l"(src), "r"(n)
                   : "memory");
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(
                       smem_u32(st + ((2 * cc + 1) * kCtxKeys + ck) * 8)),
                   "l"(src + (okc ? 8 : 0)), "r"(n)
                   : "memory");
      if (t < kCtxKeys) {
        const bool oks = ctx_locate(p, valid, j0 + t, h, seg_s, co, so);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(st + kRingScales + t * 8)),
                     "l"(p.base + (oks ? so : 0)), "r"(oks ? 8u : 0u)
                     : "memory");
        reinterpret_cast<float*>(st + kRingGv)[t] = oks ? gv_tab[seg_s] : 0.0f;
      }
    };
    for (uint32_t i = 0; i + 1 < (uint32_t)kRing; ++i) {
      if (i < n_my) issue(i);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // decoding: keys 2 kp, 2 kp + 1 of the tile, dims [16 dq, 16 dq + 16) (one scale block)
    const int kp = t & 31, dq = t >> 5;
    const int col = 2 * kp;
    // row d of a V^T tile holds its 64 keys (128 bytes, 16-byte chunks swizzled by d % 8);
    // keys 2 kp and 2 kp + 1 share one 32-bit word
    const uint32_t vt_off = (uint32_t)((col & 7) * 2);
    const uint32_t chunk = (uint32_t)(col >> 3);
    bool ok = true;
    for (uint32_t i = 0; i < n_my; ++i) {
      asm volatile("cp.async.wait_group %0;" ::"n"(kRing - 2) : "memory");  // this thread's copies of tile i
      // named barrier of the decoder warps: everyone's copies of tile i are in, tile i - 1
      // is fully read, and a wait that gave up in any warp stops all of them together
      if (named_barrier_or(1, kVThreads, !ok)) {
        ok = false;
        break;
      }
      if (i + kRing - 1 < n_my) issue(i + kRing - 1);  // into tile i - 1's stage
      asm volatile("cp.async.commit_group;" ::: "memory");
      const uint8_t* st = ring + (i % kRing) * kRingStageBytes;
      float f0[16], f1[16];
      {
        uint32_t a0, a1, b0, b1;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(a0), "=r"(a1), "=r"(b0), "=r"(b1)
                     : "r"(smem_u32(st + (dq * kCtxKeys + col) * 8)));
        const uint32_t s0 = st[kRingScales + col * 8 + dq], s1 = st[kRingScales + (col + 1) * 8 + dq];
        const float2 gv = *reinterpret_cast<const float2*>(st + kRingGv + col * 4);
        ctx_decode(a0, a1, s0, gv.x, f0);
        ctx_decode(b0, b1, s1, gv.y, f1);
      }
      const int b = i % kCtxVBufs;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&v_empty[b]), ((i / kCtxVBufs) & 1u) ^ 1u, abort_flag,
                                             limit))) {
        ok = false;  // skip the stores; the next barrier stops every decoder warp
      }
      if (ok) {
        fence_after();
        const uint32_t vb = smem_u32(vbuf + b * kVTBytes) + (uint32_t)(dq * 16 * 128) + vt_off;
#pragma unroll
        for (int d = 0; d < 16; ++d)  // dim 16 dq + d; (16 dq + d) % 8 = d % 8
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(vb + (uint32_t)(d * 128) + ((chunk ^ (uint32_t)(d & 7)) << 4)),
                       "r"(pack_bf16x2(f0[d], f1[d]))
                       : "memory");
        fence_proxy_async_smem();  // the tensor core reads V^T through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&v_full[b]));
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy into the ring outlives the loop
    if (!ok) {
      if (lane == 0) set_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    } else if (warp < kVWarp0 + 4) {
      if (__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(t_full), 0, abort_flag, limit))) {
        if (warp == kVWarp0 && lane == 0) *acc_ok = 1;
      } else {
        if (lane == 0) set_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
    }
  }

  fence_before();
  __syncthreads();
  fence_after();

  // ---------------------------------------------------------------- output
  // warps 4..7: warp w reads tensor-memory lane quarter w % 4 (query rows 32 (w % 4) ..)
  const bool reader = warp >= kVWarp0 && warp < kVWarp0 + 4;
  const int quarter = warp & 3;
  const bool have = *acc_ok != 0 && n_my > 0;
  if (p.split == 1) {
    if (reader && *acc_ok) {
      for (int g = 0; g < G; ++g) {
        const int64_t qrow = (int64_t)(qt0 + g) * kQ + quarter * 32 + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * kD + c0), r);
          if (qrow < p.Tq) {
            if (p.o_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(p.o + (qrow * p.ldo + (int64_t)h * kD + c0) * 2);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[k] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * k]), __uint_as_float(r[8 * k + 1])),
                                    pack_bf16x2(__uint_as_float(r[8 * k + 2]), __uint_as_float(r[8 * k + 3])),
                                    pack_bf16x2(__uint_as_float(r[8 * k + 4]), __uint_as_float(r[8 * k + 5])),
                                    pack_bf16x2(__uint_as_float(r[8 * k + 6]), __uint_as_float(r[8 * k + 7])));
            } else {
              uint4* dst = reinterpret_cast<uint4*>(p.o + (qrow * p.ldo + (int64_t)h * kD + c0) * 4);
#pragma unroll
              for (int k = 0; k < 8; ++k) dst[k] = make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
            }
          }
        }
      }
    }
  } else {
    const int r0 = rank * kQ / p.split, r1 = (rank + 1) * kQ / p.split;
    const uint32_t part = smem_u32(pbuf);
    for (int g = 0; g < G; ++g) {  // the same G in every CTA of the cluster
      if (reader) {
        // partial -> shared memory: row r's 16-byte chunks XOR-swizzled by r % 32
        const int row = quarter * 32 + lane;
        const uint32_t prow = part + (uint32_t)(row * kPartRowBytes);
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
          uint32_t r[32];
          if (have) {
            tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(g * kD + c0), r);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = 0u;  // no keys in this CTA's range (or a timeout)
          }
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(prow + ((((c0 >> 2) + k) ^ lane) << 4),
                         make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]));
        }
      }
      __syncthreads();
      cluster_sync_all();  // every CTA of the cluster has this tile's partial in shared memory
      for (int it = threadIdx.x; it < (r1 - r0) * (kD / 8); it += kCtxThreads) {
        const int r = r0 + it / (kD / 8), cg = it % (kD / 8);  // 8 output columns 8 cg ..
        const uint32_t a0 = part + (uint32_t)(r * kPartRowBytes) + ((uint32_t)((2 * cg) ^ (r & 31)) << 4);
        const uint32_t a1 = part + (uint32_t)(r * kPartRowBytes) + ((uint32_t)((2 * cg + 1) ^ (r & 31)) << 4);
        float acc[8];
        for (int src = 0; src < p.split; ++src) {  // cluster-rank order
          float v[8];
          uint32_t b0, b1;
          asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(b0) : "r"(a0), "r"(src));
          asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(b1) : "r"(a1), "r"(src));
          asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                       : "r"(b0)
                       : "memory");
          asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                       : "r"(b1)
                       : "memory");
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = src == 0 ? v[k] : __fadd_rn(acc[k], v[k]);
        }
        const int64_t qrow = (int64_t)(qt0 + g) * kQ + r;
        if (qrow < p.Tq) {
          if (p.o_bf16) {
            *reinterpret_cast<uint4*>(p.o + (qrow * p.ldo + (int64_t)h * kD + cg * 8) * 2) =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(p.o + (qrow * p.ldo + (int64_t)h * kD + cg * 8) * 4);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
          }
        }
      }
      cluster_sync_all();  // no CTA rewrites or releases its partial while another reads it
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kCtxTmemCols)
                 : "memory");
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

}  // namespace

cudaError_t launch_kv_scores(const KVLayout& L, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                             const void* q, int64_t tq, int64_t ldq, float scale, void* s_out, bool s_bf16,
                             int64_t ld_s, unsigned* status, cudaStream_t s) {
  if (L.head_dim != kD) return cudaErrorInvalidValue;
  ScoresParams p;
  memset(&p, 0, sizeof(p));
  p.base = L.base;
  p.off_k_codes = L.off_k_codes;
  p.off_k_scales = L.off_k_scales;
  p.off_mu = L.off_mu;
  p.off_gscale = L.off_gscale;
  p.off_tokens = L.off_tokens;
  p.slot_codes_bytes = L.slot_codes_bytes;
  p.slot_scales_bytes = L.slot_scales_bytes;
  p.heads = L.heads;
  p.n_slots = n_slots;
  int64_t acc = 0;
  for (int i = 0; i < n_slots; ++i) {
    p.slots[i] = slots[i];
    p.tokens[i] = tokens[i];
    acc += tokens[i];
    p.key_end[i] = acc;
  }
  p.Tq = tq;
  p.Tk = acc;
  p.n_items = ((acc + kKeys - 1) / kKeys) * L.heads;
  p.scale = scale;
  p.s_bf16 = s_bf16;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  if (tq == 0) return cudaSuccess;

  // queries [tq][heads * 128] bf16 (row pitch ldq elements): 64-column x 128-row boxes
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap mq;
  cuuint64_t dims[2] = {(cuuint64_t)L.heads * kD, (cuuint64_t)tq};
  cuuint64_t strides[1] = {(cuuint64_t)ldq * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kQ};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  // scores [heads][tq][ld_s]: 32-row x 128-byte boxes (64 bf16 or 32 FP32 keys), the
  // same 128-byte swizzle as the staging buffers; clipped at tq queries and Tk keys
  CUtensorMap ms;
  const cuuint64_t esz = s_bf16 ? 2 : 4;
  cuuint64_t sdims[3] = {(cuuint64_t)acc, (cuuint64_t)tq, (cuuint64_t)L.heads};
  cuuint64_t sstrides[2] = {(cuuint64_t)ld_s * esz, (cuuint64_t)ld_s * esz * (cuuint64_t)tq};
  cuuint32_t sbox[3] = {(cuuint32_t)(128 / esz), 32, 1};
  cuuint32_t sestr[3] = {1, 1, 1};
  if (fn(&ms, s_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, s_out, sdims,
         sstrides, sbox, sestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  static std::atomic<int> resident[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (resident[dev].load(std::memory_order_relaxed) == 0) {
    e = cudaFuncSetAttribute(kv_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kv_scores_kernel, kThreads, kSmemBytes);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    resident[dev].store(per_sm * sms, std::memory_order_relaxed);
  }
  // one wave of persistent CTAs, each taking items blockIdx.x, blockIdx.x + grid, ...
  const int64_t ctas = p.n_items < resident[dev].load(std::memory_order_relaxed)
                           ? p.n_items
                           : resident[dev].load(std::memory_order_relaxed);
  launch_pdl(kv_scores_kernel, dim3((unsigned)ctas, 1, 1), kThreads, kSmemBytes, s, mq, ms, p);
  return cudaGetLastError();
}

}  // namespace nvfp4

namespace nvfp4 {

cudaError_t launch_kv_context(const KVLayout& L, const int32_t* slots, const int32_t* tokens, int32_t n_slots,
                              const void* pm, int64_t tq, int64_t ld_p, void* o_out, bool o_bf16, int64_t ldo,
                              unsigned* status, cudaStream_t s) {
  if (L.head_dim != kD) return cudaErrorInvalidValue;
  ContextParams p;
  memset(&p, 0, sizeof(p));
  p.base = L.base;
  p.off_v_codes = L.off_v_codes;
  p.off_v_scales = L.off_v_scales;
  p.off_gscale = L.off_gscale;
  p.off_tokens = L.off_tokens;
  p.slot_codes_bytes = L.slot_codes_bytes;
  p.slot_scales_bytes = L.slot_scales_bytes;
  p.heads = L.heads;
  p.n_slots = n_slots;
  int64_t acc = 0;
  for (int i = 0; i < n_slots; ++i) {
    p.slots[i] = slots[i];
    p.tokens[i] = tokens[i];
    acc += tokens[i];
    p.key_end[i] = acc;
  }
  p.Tq = tq;
  p.Tk = acc;
  p.o_bf16 = o_bf16;
  p.o = static_cast<uint8_t*>(o_out);
  p.ldo = ldo;
  p.status = status;
  p.wait_limit_ns = kWaitLimitNs;
  if (tq == 0) return cudaSuccess;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  // P [heads][tq][ld_p] bf16: 64-key x 128-query boxes, 128-byte swizzle, zero-filled
  // beyond the window's keys and the query count
  CUtensorMap mp;
  cuuint64_t pdims[3] = {(cuuint64_t)acc, (cuuint64_t)tq, (cuuint64_t)L.heads};
  cuuint64_t pstrides[2] = {(cuuint64_t)ld_p * 2, (cuuint64_t)ld_p * 2 * (cuuint64_t)tq};
  cuuint32_t pbox[3] = {64, (cuuint32_t)kQ, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pm), pdims, pstrides, pbox, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  // per device: shared-memory opt-in once, and how many CTAs can be resident at once in
  // clusters of S = 1 .. kMaxSplit (0: that cluster size cannot be resident)
  static std::atomic<int> conc_cache[64][kMaxSplit + 1];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (conc_cache[dev][0].load(std::memory_order_relaxed) == 0) {
    e = cudaFuncSetAttribute(kv_context_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kCtxSmemBytes);
    if (e != cudaSuccess) return e;
    for (int c = 1; c <= kMaxSplit; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)c, 1, 1);
      cfg.blockDim = dim3(kCtxThreads, 1, 1);
      cfg.dynamicSmemBytes = kCtxSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = (unsigned)c;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kv_context_kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      if (c == 1 && n <= 0) return cudaErrorInvalidConfiguration;
      conc_cache[dev][c].store(n * c, std::memory_order_relaxed);
    }
    conc_cache[dev][0].store(1, std::memory_order_relaxed);
  }
  // G query tiles per CTA and S CTAs per cluster: the fewest waves of CTAs times the
  // longest CTA's work, in units of one P tile (128 queries x 64 keys) with a V^ tile's
  // dequantization counted as half of one.  Ties keep the smaller S.
  const int64_t n_kt = (acc + kCtxKeys - 1) / kCtxKeys;
  const int64_t n_qt = (tq + kQ - 1) / kQ;
  int best_g = (int)((n_qt + 65534) / 65535), best_s = 1;
  double best = -1.0;
  const int64_t g_min = (n_qt + 65534) / 65535;  // grid.y (query groups) is at most 65535
  if (g_min > kCtxMaxG) return cudaErrorInvalidValue;
  for (int g = (int)g_min; g <= kCtxMaxG && g <= n_qt; ++g) {
    for (int sp = 1; sp <= kMaxSplit && sp <= n_kt; ++sp) {
      const int64_t conc = conc_cache[dev][sp].load(std::memory_order_relaxed);
      if (conc <= 0) continue;
      const int64_t ctas = (int64_t)sp * ((n_qt + g - 1) / g) * L.heads;
      const int64_t waves = (ctas + conc - 1) / conc;
      const double cost = (double)waves * (double)((n_kt + sp - 1) / sp) * (g + 0.5);
      if (best < 0.0 || cost < best * (1.0 - 1e-9)) {
        best = cost;
        best_g = g;
        best_s = sp;
      }
    }
  }
  const int split = best_s;
  p.split = split;
  p.G = best_g;
  p.n_qt = (int32_t)n_qt;
  p.tiles_per_split = (n_kt + split - 1) / split;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)split, (unsigned)((n_qt + best_g - 1) / best_g), (unsigned)L.heads);
  cfg.blockDim = dim3(kCtxThreads, 1, 1);
  cfg.dynamicSmemBytes = kCtxSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)split;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kv_context_kernel, mp, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace nvfp4
