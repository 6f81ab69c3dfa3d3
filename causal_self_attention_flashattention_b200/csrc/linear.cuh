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
// sm_100a design: persistent two-CTA clusters (SM pairs) walk 256 x 256
// output tiles; the pair's tensor-core products (tcgen05 .cta_group::2)
// read half of each operand tile from each SM, so an SM loads 32 KiB of
// operands per K step of 64 instead of the 48 KiB a one-SM 128 x 256 tile
// needs. Every wait is bounded like the attention kernels'.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace linear {

constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators

struct GemmShape {
  int M, N, K;
  int f16_from;  // columns >= f16_from are written as fp16 (N: none)
};

// ---------------------------------------------------------------------------
// A two-CTA cluster computes a 256 x 256 tile of y: CTA r loads rows
// [128 r, 128 r + 128) of the tile's A rows and the same half of its W rows;
// one thread of CTA 0 issues tcgen05.mma .cta_group::2 M256 N256 K16, which
// reads both CTAs' halves and leaves each CTA's 128 rows of the tile (all 256
// columns) in that CTA's tensor memory.
//   * Warp 0 of each CTA (TMA): its A and W halves into a 6-stage ring; the
//     copies of both CTAs complete on CTA 0's `full` barrier (CTA 0 sets the
//     stage's expected bytes for the pair).
//   * Warp 1 of CTA 0 (MMA): waits on `full`, issues the pair's products and
//     commits to `empty` in both CTAs; after a tile's last K step, to
//     `acc_full` in both. Before a tile, it waits on CTA 0's `acc_empty`,
//     which counts the eight epilogue warps of the pair.
//   * Warps 2-5 of each CTA (epilogue): each thread owns one of the CTA's 128
//     rows (its TMEM lane). It reads 128 accumulator columns per tensor-memory
//     wait (32 columns per wait left the epilogue slower than the products),
//     adds the bias (one broadcast load per 8 columns), rounds to bf16 (or
//     fp16 for columns at or beyond `f16_from`) and writes its row's 64-column
//     pieces into one of the warp's two staging tiles; lane 0 stores each
//     32 x 64 tile with a TMA bulk store. Then the warp arrives (remotely,
//     from CTA 1) on CTA 0's `acc_empty`.
//     No barrier other than the bounded mbarrier waits joins the epilogue
//     warps, so a wait that gives up cannot strand the others.
constexpr int kPairBM = 256, kPairBN = 256;
constexpr int kPairStages = 6;
constexpr uint32_t kPairHalfBytes = 128 * kBK * 2;  // 16 KiB: a half tile of A or of W

constexpr int kEpiWarps = 4;
constexpr uint32_t kStageTileBytes = 32 * 128;  // 32 rows x 64 columns of 16-bit y

struct alignas(1024) PairSmem {
  uint8_t a[kPairStages][kPairHalfBytes];
  uint8_t b[kPairStages][kPairHalfBytes];
  // [epilogue warp][buffer]: 32 rows x 64 columns of y (128-byte swizzle) on
  // their way to global memory by TMA.
  uint8_t ystage[kEpiWarps][2][kStageTileBytes];
  uint64_t full[kPairStages], empty[kPairStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kPairSmemBytes = sizeof(PairSmem) + 1024;
static_assert(kPairSmemBytes <= 232448, "pair GEMM shared memory exceeds the 227 KiB per-block limit");

__host__ __device__ __forceinline__ int num_pair_tiles(const GemmShape& g) {
  return ceil_div(g.M, kPairBM) * ceil_div(g.N, kPairBN);
}

__global__ void __launch_bounds__(kThreads, 1)
linear_pair_kernel(const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_w,
                   const __grid_constant__ CUtensorMap map_y, const uint16_t* __restrict__ bias,
                   const GemmShape g) {
  extern __shared__ uint8_t smem_raw[];
  PairSmem& sm = *reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int n_clusters = static_cast<int>(gridDim.x) / 2;
  const int cid = static_cast<int>(blockIdx.x) / 2;
  const int n_tiles = num_pair_tiles(g);
  const int tiles_n = ceil_div(g.N, kPairBN);
  const int n_k = ceil_div(g.K, kBK);
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sm.full[s], 1);   // used in CTA 0: its expect-tx arrival + both CTAs' bytes
      mbar_init(&sm.empty[s], 1);  // the pair's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 8);  // used in CTA 0: the pair's eight epilogue warps
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and their tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t full0 = cluster_addr(&sm.full[0], 0);          // CTA 0's full[0]
  const uint32_t acc_empty0 = cluster_addr(&sm.acc_empty[0], 0);  // CTA 0's acc_empty[0]

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_w);
      uint32_t it = 0;
      bool ok = true;
      for (int t = cid; ok && t < n_tiles; t += n_clusters) {
        const int tm = t / tiles_n, tn = t % tiles_n;
        const int a_row = tm * kPairBM + static_cast<int>(rank) * 128;
        const int w_row = tn * kPairBN + static_cast<int>(rank) * 128;
        for (int ks = 0; ks < n_k; ++ks, ++it) {
          const int s = it % kPairStages;
          if (!mbar_wait(&sm.empty[s], ((it / kPairStages) & 1) ^ 1, kSiteLinearProducer, abort)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&sm.full[s], 4 * kPairHalfBytes);
          tma_load_2d_pair(sm.a[s], &map_a, full0 + 8u * s, ks * kBK, a_row);
          tma_load_2d_pair(sm.b[s], &map_w, full0 + 8u * s, ks * kBK, w_row);
        }
      }
      // CTA 0's full barriers count both CTAs' copies: waiting (bounded) for
      // the last phase of each means no copy of either CTA is still landing
      // (CTA 1 is held at the final cluster barrier until then).
      if (rank == 0)
        for (int s = 0; s < kPairStages; ++s)
          if (it > static_cast<uint32_t>(s))
            drain_wait(&sm.full[s], ((it - s + kPairStages - 1) / kPairStages - 1) & 1,
                       kSiteLinearProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPairBM, kPairBN, 0, 0);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = cid; ok && t < n_tiles; t += n_clusters, ++lt) {
        const uint32_t buf = lt & 1;
        if (!mbar_wait(&sm.acc_empty[buf], ((lt >> 1) & 1) ^ 1, kSiteLinearMma, abort)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * kPairBN;
        for (int ks = 0; ks < n_k; ++ks, ++it) {
          const int s = it % kPairStages;
          if (!mbar_wait(&sm.full[s], (it / kPairStages) & 1, kSiteLinearMma, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sm.a[s]), 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm.b[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss_pair(acc, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ks | kk) ? 1u : 0u);
          mma_commit_pair(&sm.empty[s]);
        }
        if (!ok) break;
        mma_commit_pair(&sm.acc_full[buf]);
      }
      // Every product has finished before either CTA frees its tensor memory.
      mma_commit_pair(&sm.drain);
      drain_wait(&sm.drain, 0, kSiteLinearMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int ew = warp - kEpiWarp0;        // this warp's staging buffers
    uint32_t lt = 0, st_cnt = 0;
    bool ok = true;
    for (int t = cid; ok && t < n_tiles; t += n_clusters, ++lt) {
      const int tm = t / tiles_n, tn = t % tiles_n;
      const uint32_t buf = lt & 1;
      const int n0 = tn * kPairBN;
      ok = mbar_wait(&sm.acc_full[buf], (lt >> 1) & 1, kSiteLinearEpilogue, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // This warp's 32 rows of the tile; rows past M are clipped by the store.
      const int row0 = tm * kPairBM + static_cast<int>(rank) * 128 + q * 32;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * kPairBN;
#pragma unroll 1
      for (int c4 = 0; c4 < kPairBN / 128; ++c4) {
        uint32_t vv[4][32];
#pragma unroll
        for (int c1 = 0; c1 < 4; ++c1) tmem_ld32(taddr + 128 * c4 + 32 * c1, vv[c1]);
        tmem_wait_ld();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // 64-column halves: one staged box each
          const int col0 = n0 + 128 * c4 + 64 * hh;
          if (col0 >= g.N) continue;  // N is a multiple of 64
          uint8_t* sb = sm.ystage[ew][st_cnt & 1];
          // The store that last read this buffer has finished reading it.
          if (lane == 0 && st_cnt >= 2) bulk_wait_group_read1();
          __syncwarp();
          const bool f16 = col0 >= g.f16_from;
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // 16-byte chunk j: columns col0 + 8j .. + 8
            const uint32_t (&v)[32] = vv[2 * hh + (j >> 2)];
            const int u = j & 3;
            // Every lane reads the same 8 bias values: one broadcast load.
            const uint4 bv = *reinterpret_cast<const uint4*>(bias + col0 + 8 * j);
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a0 = __uint_as_float(v[8 * u + 2 * e]) + __uint_as_float(bw[e] << 16);
              const float a1 = __uint_as_float(v[8 * u + 2 * e + 1]) + __uint_as_float(bw[e] & 0xFFFF0000u);
              w[e] = f16 ? pack_f16(a0, a1) : pack_bf16(a0, a1);
            }
            *reinterpret_cast<uint4*>(sb + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();  // generic-proxy writes, read by the TMA engine
          __syncwarp();
          if (lane == 0 && row0 < g.M) {  // a box wholly past M is not issued
            tma_store_2d(&map_y, sb, col0, row0);
            bulk_commit_group();
          }
          ++st_cnt;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * buf);
    }
    // Every store this warp issued has completed before the CTA exits.
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync();  // no product, copy or tensor-memory read of either CTA outstanding
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace linear
}  // namespace ga
