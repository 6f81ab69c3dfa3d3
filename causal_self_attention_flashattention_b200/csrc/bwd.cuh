// Backward kernels of causal self-attention.
//
// With P_ij = exp(s_ij - lse_i) recomputed from the stored logsumexp (flash
// attention keeps no T x T matrix: "Let's reproduce GPT-2 (124M)" video summary
// page, glossary table, row "flash attention"), the gradients are
//     dV = P^T dO,   dP = dO V^T,   dS = P o (dP - Delta),
//     dQ = scale dS K,   dK = scale dS^T Q,
// where Delta_i = sum_j P_ij dP_ij = dO_i . O_i (the row term of the softmax
// Jacobian, computed from out and dout).
//
// Three kernels, launched in this order on one stream:
//   attn_bwd_pre_kernel  Delta[b,h,t] = sum_d dO o O, fp32 (memory bound).
//   attn_bwd_dkdv_kernel one CTA per 128-key tile j: streams query tiles
//                        i >= j, accumulates dK and dV in tensor memory.
//   attn_bwd_dq_kernel   one CTA per 128-query tile i: streams key tiles
//                        j <= i, accumulates dQ in tensor memory. Nothing is
//                        accumulated through atomics, so the result is
//                        bitwise deterministic.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace bwd {

// ===========================================================================
// Delta = rowsum(dO o O)
// ===========================================================================
// Eight lanes per (b, t, h) row of 64 bf16: each lane loads 16 bytes of both
// tensors, and three shuffles finish the dot product.
__global__ void __launch_bounds__(256)
attn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                    float* __restrict__ delta, const AttnShape sh) {
  const long long rows = static_cast<long long>(sh.B) * sh.T * sh.H;
  const int sub = threadIdx.x & 7;
  // The 8 lanes of one row always take the same branch, so the shuffles only
  // name those 8 lanes: a partial last warp never waits on exited lanes.
  const unsigned group = 0xFFu << (threadIdx.x & 24);
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 3);
  for (long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
       row < rows; row += stride) {
    const uint4 a = reinterpret_cast<const uint4*>(out + row * kD)[sub];
    const uint4 g = reinterpret_cast<const uint4*>(dout + row * kD)[sub];
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 af = __bfloat1622float2(a2[e]);
      const float2 gf = __bfloat1622float2(g2[e]);
      acc = fmaf(af.x, gf.x, acc);
      acc = fmaf(af.y, gf.y, acc);
    }
    acc += __shfl_xor_sync(group, acc, 4);
    acc += __shfl_xor_sync(group, acc, 2);
    acc += __shfl_xor_sync(group, acc, 1);
    if (sub == 0) {
      const int h = static_cast<int>(row % sh.H);
      const long long bt = row / sh.H;
      const int t = static_cast<int>(bt % sh.T);
      const int b = static_cast<int>(bt / sh.T);
      delta[(static_cast<long long>(b) * sh.H + h) * sh.T + t] = acc;
    }
  }
}

constexpr int kStages = 4;
// Warps 0-7: two elementwise warpgroups. Each thread owns one row of the tile
// (its TMEM lane); warpgroup g takes the 64 columns [64g, 64g + 64).
// Warp 8: TMA producer. Warp 9: MMA issuer.
constexpr int kThreads = 320;
constexpr int kEwWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ===========================================================================
// dK, dV: one CTA per key tile
// ===========================================================================
// Per query tile i >= j (all in the transposed frame, rows = keys):
//   S^T  = K_j Q_i^T     (M128 N128 K64, both operands K-major)
//   dP^T = V_j dO_i^T    (same)
//   P^T  = exp2(S^T * scale*log2e - lse_i*log2e), zero where key > query
//   dS^T = P^T o (dP^T - Delta_i)
//   dV  += P^T dO_i      (A = P^T from tensor memory, B = dO_i MN-major)
//   dK  += dS^T Q_i      (A = dS^T from tensor memory, B = Q_i MN-major)
// Tensor memory: S^T [0,128), dP^T [128,256), P^T [256,320), dS^T [320,384)
// (bf16 pairs), dV [384,448), dK [448,512).
namespace dkdv {

struct alignas(1024) Smem {
  uint8_t k[2][kTileBytes];  // [item slot]
  uint8_t v[2][kTileBytes];
  uint8_t q[kStages][kTileBytes];
  uint8_t dout[kStages][kTileBytes];
  float lse2[kStages][kBlockM];  // lse * log2(e) of the staged query tile
  float delta[kStages][kBlockM];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t in_full[kStages], in_empty[kStages];
  uint64_t sdp_full, sdp_free, ds_full, pds_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ void decode(int k, const AttnShape& sh, int& b, int& h, int& j) {
  const int bh_count = sh.B * sh.H;
  j = k / bh_count;  // key tile 0 has the most query tiles: heaviest first
  const int bh = k % bh_count;
  b = bh / sh.H;
  h = bh % sh.H;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_qkv,
                     const __grid_constant__ CUtensorMap map_do, const float* __restrict__ lse,
                     const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv,
                     const AttnShape sh) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = sh.H * kD;
  const int n_qt = ceil_div(sh.T, kBlockM);
  const int n_items = sh.B * sh.H * n_qt;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.in_full[s], 2);  // TMA bytes + the warp's lse/Delta stores
      mbar_init(&sm.in_empty[s], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_free, kEwWarps);
    mbar_init(&sm.ds_full, kEwWarps);
    mbar_init(&sm.pds_free, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_qkv);
    tma_prefetch_desc(&map_do);
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
    // Lane 0 waits and issues the TMA copies; all 32 lanes stage the 128 lse
    // (base 2) and Delta values of each query tile next to its Q and dO tiles.
    uint32_t in_it = 0, it_cnt = 0;
    bool ok = true;
    for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
      int b, h, j;
      decode(k, sh, b, h, j);
      const int slot = it_cnt & 1;
      bool w = true;
      if (lane == 0) w = mbar_wait(&sm.kv_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteDkvProducer, abort);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.kv_full[slot], 2 * kTileBytes);
        tma_load_3d(sm.k[slot], &map_qkv, &sm.kv_full[slot], C + h * kD, j * kBlockN, b);
        tma_load_3d(sm.v[slot], &map_qkv, &sm.kv_full[slot], 2 * C + h * kD, j * kBlockN, b);
      }
      ++it_cnt;
      const size_t row_base = (static_cast<size_t>(b) * sh.H + h) * sh.T;
      for (int i = j; i < n_qt; ++i, ++in_it) {
        const int s = in_it % kStages;
        if (lane == 0) w = mbar_wait(&sm.in_empty[s], ((in_it / kStages) & 1) ^ 1, kSiteDkvProducer, abort);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = lane + 32 * e;
          const int qrow = i * kBlockM + c;
          const bool valid = qrow < sh.T;
          // Rows past T get lse = +inf, so their P is exactly 0.
          sm.lse2[s][c] = valid ? lse[row_base + qrow] * kLog2e : INFINITY;
          sm.delta[s][c] = valid ? delta[row_base + qrow] : 0.f;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.in_full[s], 2 * kTileBytes);
          tma_load_3d(sm.q[s], &map_qkv, &sm.in_full[s], h * kD, i * kBlockM, b);
          tma_load_3d(sm.dout[s], &map_do, &sm.in_full[s], h * kD, i * kBlockM, b);
          mbar_arrive(&sm.in_full[s]);
        }
      }
    }
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s)
        if (in_it > static_cast<uint32_t>(s))
          drain_wait(&sm.in_full[s], ((in_it - s + kStages - 1) / kStages - 1) & 1, kSiteDkvProducer);
      for (int s = 0; s < 2; ++s)
        if (it_cnt > static_cast<uint32_t>(s))
          drain_wait(&sm.kv_full[s], ((it_cnt - s + 1) / 2 - 1) & 1, kSiteDkvProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t t_s = tmem + 0, t_dp = tmem + 128, t_p = tmem + 256, t_ds = tmem + 320;
      const uint32_t t_dv = tmem + 384, t_dk = tmem + 448;
      uint32_t in_it = 0, it_cnt = 0, sdp_cnt = 0, ds_cnt = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x, ++it_cnt) {
        int b, h, j;
        decode(k, sh, b, h, j);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.kv_full[slot], (it_cnt >> 1) & 1, kSiteDkvMma, abort)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[slot]), 16, 1024);
        const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[slot]), 16, 1024);
        const int n_i = n_qt - j;
        // Issues S^T and dP^T for the idx-th query tile of this item.
        auto issue_sdp = [&](uint32_t it_idx) -> bool {
          const int s = it_idx % kStages;
          if (!mbar_wait(&sm.in_full[s], (it_idx / kStages) & 1, kSiteDkvMma, abort)) return false;
          if (sdp_cnt > 0 && !mbar_wait(&sm.sdp_free, (sdp_cnt - 1) & 1, kSiteDkvMma, abort))
            return false;
          tc_fence_after();
          const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.q[s]), 16, 1024);
          const uint64_t odesc = smem_desc_sw128(smem_u32(sm.dout[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) mma_ss(t_s, kdesc + 2 * kk, qdesc + 2 * kk, idesc_s, kk > 0);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) mma_ss(t_dp, vdesc + 2 * kk, odesc + 2 * kk, idesc_s, kk > 0);
          mma_commit(&sm.sdp_full);
          ++sdp_cnt;
          return true;
        };
        if (!issue_sdp(in_it)) { ok = false; break; }
        for (int n = 0; n < n_i; ++n) {
          const uint32_t cur = in_it + n;
          if (n + 1 < n_i && !issue_sdp(cur + 1)) { ok = false; break; }
          if (!mbar_wait(&sm.ds_full, ds_cnt & 1, kSiteDkvMma, abort)) { ok = false; break; }
          ++ds_cnt;
          tc_fence_after();
          const int s = cur % kStages;
          const uint64_t qdesc_mn = smem_desc_sw128(smem_u32(sm.q[s]), 128 * 128, 1024);
          const uint64_t odesc_mn = smem_desc_sw128(smem_u32(sm.dout[s]), 128 * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < kBlockM / 16; ++kk)
            mma_ts(t_dv, t_p + 8 * kk, odesc_mn + 128 * kk, idesc_acc, (n > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kBlockM / 16; ++kk)
            mma_ts(t_dk, t_ds + 8 * kk, qdesc_mn + 128 * kk, idesc_acc, (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.pds_free);
          mma_commit(&sm.in_empty[s]);
        }
        if (!ok) break;
        in_it += n_i;
        mma_commit(&sm.kv_empty[slot]);
      }
      mma_commit(&sm.drain);
      drain_wait(&sm.drain, 0, kSiteDkvMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- elementwise WGs
    const int r = ((warp & 3) << 5) + lane;  // key row within the tile = TMEM lane
    const int g = warp >> 2;                 // query columns [64g, 64g + 64)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t t_s = tmem + lane_base + 64 * g, t_dp = tmem + lane_base + 128 + 64 * g;
    const uint32_t t_p = tmem + lane_base + 256 + 32 * g, t_ds = tmem + lane_base + 320 + 32 * g;
    const uint32_t t_dv = tmem + lane_base + 384 + 32 * g, t_dk = tmem + lane_base + 448 + 32 * g;
    uint32_t sdp_cnt = 0, pds_cnt = 0, in_it = 0;
    bool ok = true;
    for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
      int b, h, j;
      decode(k, sh, b, h, j);
      for (int i = j; i < n_qt; ++i, ++in_it) {
        // The stage's in_full phase (already complete: the MMA warp waited on
        // it) makes the producer's lse/Delta stores visible to this thread.
        ok = mbar_wait(&sm.in_full[in_it % kStages], (in_it / kStages) & 1, kSiteDkvSoftmax, abort);
        ok = ok && mbar_wait(&sm.sdp_full, sdp_cnt & 1, kSiteDkvSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sdp_cnt;
        tc_fence_after();
        const bool diag = (i == j);
        const float* l2 = sm.lse2[in_it % kStages] + 64 * g;
        const float* dl = sm.delta[in_it % kStages] + 64 * g;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {  // 32 query columns at a time
          uint32_t sv[32], dv[32];
          tmem_ld32(t_s + 32 * half, sv);
          tmem_ld32(t_dp + 32 * half, dv);
          tmem_wait_ld();
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sdp_free);
          }
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 L = reinterpret_cast<const float4*>(l2 + 32 * half)[c4];
            const float4 Dl = reinterpret_cast<const float4*>(dl + 32 * half)[c4];
            const float lv[4] = {L.x, L.y, L.z, L.w};
            const float dlv[4] = {Dl.x, Dl.y, Dl.z, Dl.w};
            float p[4], ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              float x = fmaf(__uint_as_float(sv[c]), sh.scale_log2, -lv[e]);
              if (diag && (64 * g + 32 * half + c) < r) x = -INFINITY;  // key r after query
              p[e] = ex2(x);
              ds[e] = p[e] * (__uint_as_float(dv[c]) - dlv[e]);
            }
            pp[2 * c4] = pack_bf16_fast(p[0], p[1]);
            pp[2 * c4 + 1] = pack_bf16_fast(p[2], p[3]);
            dd[2 * c4] = pack_bf16_fast(ds[0], ds[1]);
            dd[2 * c4 + 1] = pack_bf16_fast(ds[2], ds[3]);
          }
          if (half == 0 && i > j) {
            // The previous tile's dV/dK MMAs must be done reading P^T, dS^T.
            ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteDkvSoftmax, abort);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            ++pds_cnt;
            tc_fence_after();
          }
          tmem_st16(t_p + 16 * half, pp);
          tmem_st16(t_ds + 16 * half, dd);
        }
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
      }
      if (!ok) break;
      // The last tile's pds_free phase: dV and dK are complete.
      ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteDkvSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++pds_cnt;
      tc_fence_after();
      // Warpgroup g stores d columns [32g, 32g + 32) of dV and dK.
      uint32_t av[32], ak[32];
      tmem_ld32(t_dv, av);
      tmem_ld32(t_dk, ak);
      tmem_wait_ld();
      tc_fence_before();
      const int key = j * kBlockN + r;
      if (key < sh.T) {
        __nv_bfloat16* base = dqkv + ((static_cast<size_t>(b) * sh.T + key) * 3) * C + h * kD + 32 * g;
        uint4* dst_v = reinterpret_cast<uint4*>(base + 2 * C);
        uint4* dst_k = reinterpret_cast<uint4*>(base + C);
        const float sc = sh.scale;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          dst_v[v] = make_uint4(pack_bf16(__uint_as_float(av[8 * v]), __uint_as_float(av[8 * v + 1])),
                                pack_bf16(__uint_as_float(av[8 * v + 2]), __uint_as_float(av[8 * v + 3])),
                                pack_bf16(__uint_as_float(av[8 * v + 4]), __uint_as_float(av[8 * v + 5])),
                                pack_bf16(__uint_as_float(av[8 * v + 6]), __uint_as_float(av[8 * v + 7])));
          dst_k[v] = make_uint4(
              pack_bf16(__uint_as_float(ak[8 * v]) * sc, __uint_as_float(ak[8 * v + 1]) * sc),
              pack_bf16(__uint_as_float(ak[8 * v + 2]) * sc, __uint_as_float(ak[8 * v + 3]) * sc),
              pack_bf16(__uint_as_float(ak[8 * v + 4]) * sc, __uint_as_float(ak[8 * v + 5]) * sc),
              pack_bf16(__uint_as_float(ak[8 * v + 6]) * sc, __uint_as_float(ak[8 * v + 7]) * sc));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace dkdv

// ===========================================================================
// dQ: one CTA per query tile
// ===========================================================================
// Per key tile j <= i:
//   S  = Q_i K_j^T    (M128 N128 K64, K-major operands)
//   dP = dO_i V_j^T   (same)
//   P  = exp2(S * scale*log2e - lse*log2e) (row constants live in registers),
//        zero where key > query
//   dS = P o (dP - Delta)
//   dQ += dS K_j      (A = dS from tensor memory, B = K_j MN-major)
// Tensor memory: S [0,128), dP [128,256), dS double-buffered [256,320) and
// [320,384) (bf16 pairs), dQ [384,448).
namespace dq {

struct alignas(1024) Smem {
  uint8_t q[2][kTileBytes];  // [item slot]
  uint8_t dout[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t in_full[2], in_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sdp_full, sdp_free, ds_full, acc_done;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ void decode(int k, const AttnShape& sh, int n_qt, int& b, int& h,
                                       int& i) {
  const int bh_count = sh.B * sh.H;
  i = n_qt - 1 - k / bh_count;  // the last query tile sees the most keys: heaviest first
  const int bh = k % bh_count;
  b = bh / sh.H;
  h = bh % sh.H;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap map_qkv,
                   const __grid_constant__ CUtensorMap map_do, const float* __restrict__ lse,
                   const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv,
                   const AttnShape sh) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = sh.H * kD;
  const int n_qt = ceil_div(sh.T, kBlockM);
  const int n_items = sh.B * sh.H * n_qt;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.in_full[s], 1);
      mbar_init(&sm.in_empty[s], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_free, kEwWarps);
    mbar_init(&sm.ds_full, kEwWarps);
    mbar_init(&sm.acc_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_qkv);
    tma_prefetch_desc(&map_do);
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
      uint32_t kv_it = 0, it_cnt = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
        int b, h, i;
        decode(k, sh, n_qt, b, h, i);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.in_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteDqProducer, abort)) break;
        mbar_arrive_expect_tx(&sm.in_full[slot], 2 * kTileBytes);
        tma_load_3d(sm.q[slot], &map_qkv, &sm.in_full[slot], h * kD, i * kBlockM, b);
        tma_load_3d(sm.dout[slot], &map_do, &sm.in_full[slot], h * kD, i * kBlockM, b);
        ++it_cnt;
        for (int j = 0; j <= i; ++j, ++kv_it) {
          const int s = kv_it % kStages;
          if (!mbar_wait(&sm.kv_empty[s], ((kv_it / kStages) & 1) ^ 1, kSiteDqProducer, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kTileBytes);
          tma_load_3d(sm.k[s], &map_qkv, &sm.kv_full[s], C + h * kD, j * kBlockN, b);
          tma_load_3d(sm.v[s], &map_qkv, &sm.kv_full[s], 2 * C + h * kD, j * kBlockN, b);
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (kv_it > static_cast<uint32_t>(s))
          drain_wait(&sm.kv_full[s], ((kv_it - s + kStages - 1) / kStages - 1) & 1, kSiteDqProducer);
      for (int s = 0; s < 2; ++s)
        if (it_cnt > static_cast<uint32_t>(s))
          drain_wait(&sm.in_full[s], ((it_cnt - s + 1) / 2 - 1) & 1, kSiteDqProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t t_s = tmem + 0, t_dp = tmem + 128, t_ds0 = tmem + 256, t_dq = tmem + 384;
      uint32_t kv_it = 0, it_cnt = 0, sdp_cnt = 0, ds_cnt = 0;
      bool ok = true;
      for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x, ++it_cnt) {
        int b, h, i;
        decode(k, sh, n_qt, b, h, i);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.in_full[slot], (it_cnt >> 1) & 1, kSiteDqMma, abort)) { ok = false; break; }
        tc_fence_after();
        const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.q[slot]), 16, 1024);
        const uint64_t odesc = smem_desc_sw128(smem_u32(sm.dout[slot]), 16, 1024);
        const int n_j = i + 1;
        auto issue_sdp = [&](uint32_t it_idx) -> bool {
          const int s = it_idx % kStages;
          if (!mbar_wait(&sm.kv_full[s], (it_idx / kStages) & 1, kSiteDqMma, abort)) return false;
          if (sdp_cnt > 0 && !mbar_wait(&sm.sdp_free, (sdp_cnt - 1) & 1, kSiteDqMma, abort))
            return false;
          tc_fence_after();
          const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[s]), 16, 1024);
          const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) mma_ss(t_s, qdesc + 2 * kk, kdesc + 2 * kk, idesc_s, kk > 0);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) mma_ss(t_dp, odesc + 2 * kk, vdesc + 2 * kk, idesc_s, kk > 0);
          mma_commit(&sm.sdp_full);
          ++sdp_cnt;
          return true;
        };
        if (!issue_sdp(kv_it)) { ok = false; break; }
        for (int n = 0; n < n_j; ++n) {
          const uint32_t cur = kv_it + n;
          if (n + 1 < n_j && !issue_sdp(cur + 1)) { ok = false; break; }
          if (!mbar_wait(&sm.ds_full, ds_cnt & 1, kSiteDqMma, abort)) { ok = false; break; }
          const uint32_t t_ds = t_ds0 + 64 * (ds_cnt & 1);
          ++ds_cnt;
          tc_fence_after();
          const int s = cur % kStages;
          const uint64_t kdesc_mn = smem_desc_sw128(smem_u32(sm.k[s]), 128 * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk)
            mma_ts(t_dq, t_ds + 8 * kk, kdesc_mn + 128 * kk, idesc_acc, (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.kv_empty[s]);
        }
        if (!ok) break;
        kv_it += n_j;
        mma_commit(&sm.acc_done);
        mma_commit(&sm.in_empty[slot]);
      }
      mma_commit(&sm.drain);
      drain_wait(&sm.drain, 0, kSiteDqMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- elementwise WGs
    const int r = ((warp & 3) << 5) + lane;  // query row within the tile = TMEM lane
    const int g = warp >> 2;                 // key columns [64g, 64g + 64)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t t_s = tmem + lane_base + 64 * g, t_dp = tmem + lane_base + 128 + 64 * g;
    const uint32_t t_ds0 = tmem + lane_base + 256 + 32 * g, t_dq = tmem + lane_base + 384 + 32 * g;
    uint32_t sdp_cnt = 0, acc_cnt = 0, ds_cnt = 0;
    bool ok = true;
    for (int k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
      int b, h, i;
      decode(k, sh, n_qt, b, h, i);
      const int row = i * kBlockM + r;
      const bool valid = row < sh.T;
      const size_t lrow = (static_cast<size_t>(b) * sh.H + h) * sh.T + row;
      const float lse2 = valid ? lse[lrow] * kLog2e : INFINITY;
      const float dlt = valid ? delta[lrow] : 0.f;
      for (int j = 0; j <= i; ++j) {
        ok = mbar_wait(&sm.sdp_full, sdp_cnt & 1, kSiteDqSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sdp_cnt;
        tc_fence_after();
        const bool diag = (j == i);
        const uint32_t t_ds = t_ds0 + 64 * (ds_cnt & 1);
        ++ds_cnt;
        uint32_t sv[64], dv[64];
        tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(sv));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
        tmem_ld32(t_dp, *reinterpret_cast<uint32_t(*)[32]>(dv));
        tmem_ld32(t_dp + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sdp_free);
        uint32_t dd[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          float ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 2 * c2 + e;
            float x = fmaf(__uint_as_float(sv[c]), sh.scale_log2, -lse2);
            if (diag && (64 * g + c) > r) x = -INFINITY;  // key after query
            const float p = ex2(x);
            ds[e] = p * (__uint_as_float(dv[c]) - dlt);
          }
          dd[c2] = pack_bf16_fast(ds[0], ds[1]);
        }
        tmem_st32(t_ds, dd);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
      }
      if (!ok) break;
      ok = mbar_wait(&sm.acc_done, acc_cnt & 1, kSiteDqSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++acc_cnt;
      tc_fence_after();
      // Warpgroup g stores d columns [32g, 32g + 32) of dQ.
      uint32_t a[32];
      tmem_ld32(t_dq, a);
      tmem_wait_ld();
      tc_fence_before();
      if (valid) {
        const float sc = sh.scale;
        uint4* dst = reinterpret_cast<uint4*>(dqkv + ((static_cast<size_t>(b) * sh.T + row) * 3) * C +
                                              h * kD + 32 * g);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[v] = make_uint4(
              pack_bf16(__uint_as_float(a[8 * v]) * sc, __uint_as_float(a[8 * v + 1]) * sc),
              pack_bf16(__uint_as_float(a[8 * v + 2]) * sc, __uint_as_float(a[8 * v + 3]) * sc),
              pack_bf16(__uint_as_float(a[8 * v + 4]) * sc, __uint_as_float(a[8 * v + 5]) * sc),
              pack_bf16(__uint_as_float(a[8 * v + 6]) * sc, __uint_as_float(a[8 * v + 7]) * sc));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace dq
}  // namespace bwd
}  // namespace ga
