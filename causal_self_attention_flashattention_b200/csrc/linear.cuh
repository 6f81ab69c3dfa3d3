// The dense layers on either side of attention in a GPT-2 block:
//     c_attn:  qkv = x W_attn^T + b_attn   (M, C) -> (M, 3C)
//     c_proj:  y   = out W_proj^T + b_proj (M, C) -> (M, C)
// ("Andrej Karpathy - Lets reproduce GPT 2 124M" video description, chapter
// 00:13:47, the GPT-2 nn.Module; "Comment recréer GPT2 en 4 heures ?",
// section 5, the block rearrangement that makes theory and practice meet).
// The row-major (M, 3C) output of c_attn is exactly the packed
// (B, T, 3, H, D) q, k, v the attention kernels read, and the attention
// output (B, T, H, D) is exactly the (M, C) input of c_proj, so neither needs
// a layout pass: both are this one GEMM, y = A W^T + bias, written straight
// into the layout the next step reads.
//
// sm_100a design: a persistent CTA per SM walks 128 x 256 output tiles.
//   * Warp 0 (TMA): streams 128 x 64 tiles of A and 256 x 64 tiles of W
//     (128-byte swizzle, rows past M or N read as zero) through a 4-stage
//     ring.
//   * Warp 1 (MMA, one thread): four tcgen05.mma M128 N256 K16 per stage into
//     one of two 256-column fp32 accumulators in tensor memory, so the next
//     tile's products run while the previous tile's epilogue reads out.
//   * Warps 2-5 (epilogue): each thread owns one output row (its TMEM lane),
//     adds the bias (read as one broadcast load per 8 columns), rounds to bf16
//     (or fp16 for columns at or beyond `f16_from`) and stores 16-byte pieces
//     of its row. No barrier other than the bounded mbarrier waits joins the
//     epilogue warps, so a wait that gives up cannot strand the others.
// Every wait is bounded like the attention kernels'.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace linear {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
constexpr uint32_t kABytes = kBM * kBK * 2, kBBytes = kBN * kBK * 2;

struct alignas(1024) Smem {
  uint8_t a[kStages][kABytes];
  uint8_t b[kStages][kBBytes];
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "linear shared memory exceeds the 227 KiB per-block limit");

struct GemmShape {
  int M, N, K;
  int tiles_n;   // ceil(N / kBN)
  int f16_from;  // columns >= f16_from are written as fp16 (N: none)
};

__device__ __forceinline__ int num_tiles(const GemmShape& g) {
  return ceil_div(g.M, kBM) * g.tiles_n;
}

__global__ void __launch_bounds__(kThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
              const uint16_t* __restrict__ bias, uint16_t* __restrict__ y,
              const GemmShape g) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = num_tiles(g);
  const int n_k = ceil_div(g.K, kBK);
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_w);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int tm = t / g.tiles_n, tn = t % g.tiles_n;
        for (int ks = 0; ks < n_k; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, kSiteLinearProducer, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], kABytes + kBBytes);
          tma_load_2d(sm.a[s], &map_a, &sm.full[s], ks * kBK, tm * kBM);
          tma_load_2d(sm.b[s], &map_w, &sm.full[s], ks * kBK, tn * kBN);
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (it > static_cast<uint32_t>(s))
          drain_wait(&sm.full[s], ((it - s + kStages - 1) / kStages - 1) & 1, kSiteLinearProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
        const uint32_t buf = lt & 1;
        if (!mbar_wait(&sm.acc_empty[buf], ((lt >> 1) & 1) ^ 1, kSiteLinearMma, abort)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * kBN;
        for (int ks = 0; ks < n_k; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sm.full[s], (it / kStages) & 1, kSiteLinearMma, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sm.a[s]), 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.b[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss(acc, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) ? 1u : 0u);
          mma_commit(&sm.empty[s]);
        }
        if (!ok) break;
        mma_commit(&sm.acc_full[buf]);
      }
      mma_commit(&sm.drain);
      drain_wait(&sm.drain, 0, kSiteLinearMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;            // row within the tile
    uint32_t lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++lt) {
      const int tm = t / g.tiles_n, tn = t % g.tiles_n;
      const uint32_t buf = lt & 1;
      const int n0 = tn * kBN;
      ok = mbar_wait(&sm.acc_full[buf], (lt >> 1) & 1, kSiteLinearEpilogue, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int row = tm * kBM + r;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * kBN;
      uint16_t* yrow = y + static_cast<size_t>(row) * g.N;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + 32 * c, v);
        tmem_wait_ld();
        const int col0 = n0 + 32 * c;
        if (row < g.M) {
          const bool f16 = col0 >= g.f16_from;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = col0 + 8 * u;
            if (col < g.N) {
              // Every lane reads the same 8 bias values: one broadcast load.
              const uint4 bv = *reinterpret_cast<const uint4*>(bias + col);
              const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a0 = __uint_as_float(v[8 * u + 2 * e]) + __uint_as_float(bw[e] << 16);
                const float a1 = __uint_as_float(v[8 * u + 2 * e + 1]) + __uint_as_float(bw[e] & 0xFFFF0000u);
                w[e] = f16 ? pack_f16(a0, a1) : pack_bf16(a0, a1);
              }
              *reinterpret_cast<uint4*>(yrow + col) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace linear
}  // namespace ga
