// Fused backward: dK, dV and dQ from one pass over the causal tiles.
//
// The split backward (dK/dV kernel, then dQ kernel) computes S, P, dP and dS
// for every tile twice. Here one CTA per key tile j computes them once per
// query tile i >= j and issues all three accumulating products:
//     dV_j += P^T_ij dO_i,   dK_j += dS^T_ij Q_i,   dQ_ij = dS_ij K_j.
// dV and dK stay in tensor memory for the whole item, as in the dK/dV kernel.
// dQ_i sums over key tiles 0..i, which different CTAs own, so each partial
// dQ_ij goes to an fp32 buffer in the workspace in a fixed order: key tile j
// adds only after key tiles 0..j-1 have (a per-query-tile counter that every
// contributing warp increments), so the sum, and dq, are bitwise the same on
// every run. Key tile i is the last contributor to dQ_i; it scales the sum and
// writes dq (bf16) itself, so no extra pass runs.
//
// Layout of the work:
//   * A CTA walks its query tiles from the last to the diagonal one (i = j),
//     so the diagonal tile, whose dQ contribution comes last, is processed
//     last. CTAs take items (b, h, j) in index order, j-major: the owner of
//     (b, h, j-1) always has a smaller item index, so it runs in the same or
//     an earlier round of the persistent grid and never waits on (b, h, j).
//   * dS^T is written to shared memory once, 128-byte swizzled. The same bytes
//     are the K-major A operand of dK += dS^T Q (rows = keys) and the MN-major
//     A operand of dQ = dS K (rows = queries); P^T goes to tensor memory for
//     dV += P^T dO as in the dK/dV kernel.
//   * A dQ warpgroup (warps 19-22) reads each tile's dQ product out of
//     tensor memory as soon as it is done, frees the columns for the next
//     tile's product, and then adds the rows to the buffer. The counters of
//     an item's query tiles are released together when the item ends: one
//     GPU-scope fence per item instead of one per tile (each costs
//     microseconds). The owner of (b, h, j-1) has a smaller item index, so it
//     normally finished before (b, h, j) starts and nothing waits. Nothing
//     else in the CTA waits on another CTA, so the waits cannot form a cycle.
//
// Warps: 0-15 elementwise (four warpgroups, 32 query columns each), 16 TMA,
// 17 S/dP products (owns tensor memory), 18 dV/dK/dQ products, 19-22 dQ sums.
// Tensor memory: S'^T [0,128), dP'^T [128,256), P^T [256,320) (bf16 pairs),
// dQ [320,384), dV [384,448), dK [448,512).
#pragma once

#include "bwd.cuh"

namespace ga {
namespace bwd {
namespace fused {

using dkdv::bf16_pair;
using dkdv::ext_row;
using dkdv::kExtBytes;
using dkdv::kExtLbo;
using dkdv::kExtSbo;
using dkdv::split3_bf16;

constexpr int kInStages = 3;  // Q/dO ring (the dS^T tile takes the fourth stage's room)
constexpr int kDqWarp0 = 19;  // warps 19-22: one per TMEM lane quarter (warp % 4)
constexpr int kFusedThreads = 23 * 32;

struct alignas(1024) Smem {
  uint8_t k[2][kTileBytes];  // [item slot]
  uint8_t v[2][kTileBytes];
  uint8_t q[kInStages][kTileBytes];
  uint8_t dout[kInStages][kTileBytes];
  uint8_t ds[2][kTileBytes];  // dS^T, query columns [64c, 64c + 64) in ds[c]
  uint8_t ext_a[2][kExtBytes];
  uint8_t ext_b[kInStages][kExtBytes];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t in_full[kInStages], in_empty[kInStages];
  uint64_t sdp_full, sdp_free, ds_full, pds_free;
  uint64_t dq_full, dq_free;  // dQ product of a tile done / read out of tensor memory
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "fused backward shared memory exceeds the 227 KiB limit");

// Workspace layout (bytes): Delta fp32 (B,H,T) | dQ sums | counters u32
// (B,H,n_qt). Offsets are 256-byte aligned. The dQ sums of one 128-row query
// tile are 16 column chunks of 128 float4, chunk-major: element (row r, d
// columns [4t, 4t+4)) at float4 index t*128 + r, so a warp's 32 rows of one
// chunk are 512 contiguous bytes.
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__host__ __device__ inline size_t ws_dq_offset(int B, int T, int H) {
  return align256(static_cast<size_t>(B) * H * T * sizeof(float));
}
__host__ __device__ inline size_t ws_cnt_offset(int B, int T, int H) {
  return ws_dq_offset(B, T, H) +
         align256(static_cast<size_t>(B) * H * ceil_div(T, kBlockM) * kBlockM * kD * sizeof(float));
}
__host__ __device__ inline size_t ws_bytes(int B, int T, int H) {
  return ws_cnt_offset(B, T, H) + align256(static_cast<size_t>(B) * H * ceil_div(T, kBlockM) * 4);
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (2 s, like the mbarrier waits) until *p >= target.
__device__ __forceinline__ bool wait_counter(const uint32_t* p, uint32_t target, uint32_t site,
                                             volatile int* abort) {
  if (ld_acquire_gpu(p) >= target) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(128);
    if (ld_acquire_gpu(p) >= target) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitTimeoutNs) {
        record_failure(site);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// One dQ-warp's share of the ordered sum for query tile i, key tile j: the
// rows of its TMEM lane quarter, all 64 d columns (`q`, fp32 bits). Waits
// until key tiles 0..j-1 have added (4 warps each), then adds (j == 0
// stores), or, for the last contributor j == i, scales the total and writes
// dq as bf16. Returns false if the wait gave up.
__device__ __forceinline__ bool add_dq(uint32_t (&q)[64], float* __restrict__ dq_sum,
                                       const uint32_t* cnt, __nv_bfloat16* __restrict__ dqkv,
                                       int b, int h, int i, int j, int r, int lane, int n_qt,
                                       int C, const AttnShape& sh, volatile int* abort) {
  bool ok = true;
  if (j > 0 && lane == 0) ok = wait_counter(cnt, 4u * j, kSiteFusedDq, abort);
  ok = __shfl_sync(0xffffffffu, ok, 0);  // orders the other lanes' loads after lane 0's acquire
  if (!ok) return false;
  const int row = i * kBlockM + r;
  if (row >= sh.T) return true;
  float4* acc = reinterpret_cast<float4*>(dq_sum) +
                ((static_cast<size_t>(b) * sh.H + h) * n_qt + i) * (16 * kBlockM) + r;
  if (j > 0) {
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const float4 x = __ldcg(acc + t * kBlockM);  // L2: written by other SMs
      float v0 = __uint_as_float(q[4 * t]), v1 = __uint_as_float(q[4 * t + 1]);
      float v2 = __uint_as_float(q[4 * t + 2]), v3 = __uint_as_float(q[4 * t + 3]);
      add2(v0, v1, x.x, x.y);
      add2(v2, v3, x.z, x.w);
      q[4 * t] = __float_as_uint(v0);
      q[4 * t + 1] = __float_as_uint(v1);
      q[4 * t + 2] = __float_as_uint(v2);
      q[4 * t + 3] = __float_as_uint(v3);
    }
  }
  if (j == i) {
    const float s = sh.scale;
    uint4* dst = reinterpret_cast<uint4*>(dqkv + ((static_cast<size_t>(b) * sh.T + row) * 3) * C + h * kD);
#pragma unroll
    for (int t = 0; t < 8; ++t)
      dst[t] = make_uint4(
          pack_bf16(__uint_as_float(q[8 * t]) * s, __uint_as_float(q[8 * t + 1]) * s),
          pack_bf16(__uint_as_float(q[8 * t + 2]) * s, __uint_as_float(q[8 * t + 3]) * s),
          pack_bf16(__uint_as_float(q[8 * t + 4]) * s, __uint_as_float(q[8 * t + 5]) * s),
          pack_bf16(__uint_as_float(q[8 * t + 6]) * s, __uint_as_float(q[8 * t + 7]) * s));
  } else {
#pragma unroll
    for (int t = 0; t < 16; ++t)
      __stcg(acc + t * kBlockM, make_float4(__uint_as_float(q[4 * t]), __uint_as_float(q[4 * t + 1]),
                                  __uint_as_float(q[4 * t + 2]), __uint_as_float(q[4 * t + 3])));
  }
  return true;
}

// Writes this thread's 32 dS^T values (key row r, query columns [32g, 32g+32))
// into the 128-byte-swizzled tile: 16-byte chunk c of row r sits at chunk
// position c ^ (r & 7), rows 128 bytes apart, 8-row groups 1024 bytes apart.
__device__ __forceinline__ void store_ds_row(Smem& sm, const uint32_t (&dd)[16], int r, int g) {
  uint8_t* row = sm.ds[g >> 1] + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int c = 4 * (g & 1) + t;
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
        make_uint4(dd[4 * t], dd[4 * t + 1], dd[4 * t + 2], dd[4 * t + 3]);
  }
}

__device__ __forceinline__ void decode(int k, const AttnShape& sh, int& b, int& h, int& j) {
  const int bh_count = sh.B * sh.H;
  j = k / bh_count;  // j-major: key tile 0 (most query tiles) first
  const int bh = k % bh_count;
  b = bh / sh.H;
  h = bh % sh.H;
}

__global__ void __launch_bounds__(kFusedThreads, 1)
attn_bwd_fused_kernel(const __grid_constant__ CUtensorMap map_qkv,
                      const __grid_constant__ CUtensorMap map_do, const float* __restrict__ lse,
                      const float* __restrict__ delta, float* __restrict__ dq_sum,
                      uint32_t* __restrict__ counters, __nv_bfloat16* __restrict__ dqkv,
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
    for (int s = 0; s < kInStages; ++s) {
      mbar_init(&sm.in_full[s], 2);  // TMA bytes + the producer warp's B_ext stores
      mbar_init(&sm.in_empty[s], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_free, kEwWarps);
    mbar_init(&sm.ds_full, kEwWarps);
    mbar_init(&sm.pds_free, 1);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_free, 4);
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  // Constant A_ext tiles (terms 0-2 pick -lse/scale, 3-5 pick -Delta) and the
  // zero second core matrix of every B_ext tile, as in the dK/dV kernel.
  for (int idx = threadIdx.x; idx < 2 * kBlockN; idx += kFusedThreads) {
    const int which = idx / kBlockN, rr = idx % kBlockN;
    uint4* a = reinterpret_cast<uint4*>(sm.ext_a[which] + ext_row(rr));
    a[0] = which == 0 ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u)
                      : make_uint4(0u, 0x3F800000u, 0x3F803F80u, 0u);
    a[kExtLbo / 16] = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int idx = threadIdx.x; idx < kInStages * static_cast<int>(kExtBytes / 16); idx += kFusedThreads)
    reinterpret_cast<uint4*>(&sm.ext_b[0][0])[idx] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
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
    // Lane 0 waits and issues the TMA copies; all 32 lanes write the query
    // tile's B_ext (-lse/scale and -Delta as bf16 terms) next to its Q and dO.
    const float inv_scale = 1.f / sh.scale;
    uint32_t in_it = 0, it_cnt = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
      const int k = snake_item(rnd, gridDim.x, blockIdx.x);
      if (k >= n_items) continue;
      int b, h, j;
      decode(k, sh, b, h, j);
      const int slot = it_cnt & 1;
      bool w = true;
      if (lane == 0) w = mbar_wait(&sm.kv_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteFusedProducer, abort);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.kv_full[slot], 2 * kTileBytes);
        tma_load_3d(sm.k[slot], &map_qkv, &sm.kv_full[slot], C + h * kD, j * kBlockN, b);
        tma_load_3d(sm.v[slot], &map_qkv, &sm.kv_full[slot], 2 * C + h * kD, j * kBlockN, b);
      }
      ++it_cnt;
      const size_t row_base = (static_cast<size_t>(b) * sh.H + h) * sh.T;
      for (int i = n_qt - 1; i >= j; --i, ++in_it) {
        const int s = in_it % kInStages;
        if (lane == 0)
          w = mbar_wait(&sm.in_empty[s], ((in_it / kInStages) & 1) ^ 1, kSiteFusedProducer, abort);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = lane + 32 * e;
          const int qrow = i * kBlockM + c;
          const bool valid = qrow < sh.T;
          // Rows past T get -1e30 (finite, so 0 x term stays 0 in the other
          // product): their P underflows to exactly 0.
          const float vl = valid ? -lse[row_base + qrow] * inv_scale : -1e30f;
          const float vd = valid ? -delta[row_base + qrow] : 0.f;
          __nv_bfloat16 l1, l2, l3, d1, d2, d3;
          split3_bf16(vl, l1, l2, l3);
          split3_bf16(vd, d1, d2, d3);
          *reinterpret_cast<uint4*>(sm.ext_b[s] + ext_row(c)) =
              make_uint4(bf16_pair(l1, l2), bf16_pair(l3, d1), bf16_pair(d2, d3), 0u);
        }
        fence_proxy_async_smem();
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
      for (int s = 0; s < kInStages; ++s)
        if (in_it > static_cast<uint32_t>(s))
          drain_wait(&sm.in_full[s], ((in_it - s + kInStages - 1) / kInStages - 1) & 1,
                     kSiteFusedProducer);
      for (int s = 0; s < 2; ++s)
        if (it_cnt > static_cast<uint32_t>(s))
          drain_wait(&sm.kv_full[s], ((it_cnt - s + 1) / 2 - 1) & 1, kSiteFusedProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // S'^T and dP'^T (with the extra K step) for every query tile.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint64_t aext_s = smem_desc_noswizzle(smem_u32(sm.ext_a[0]), kExtLbo, kExtSbo);
      const uint64_t aext_dp = smem_desc_noswizzle(smem_u32(sm.ext_a[1]), kExtLbo, kExtSbo);
      const uint32_t t_s = tmem + 0, t_dp = tmem + 128;
      uint32_t in_it = 0, it_cnt = 0, sdp_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, j;
        decode(k, sh, b, h, j);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.kv_full[slot], (it_cnt >> 1) & 1, kSiteFusedMma, abort)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[slot]), 16, 1024);
        const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[slot]), 16, 1024);
        const int n_i = n_qt - j;
        for (int n = 0; n < n_i; ++n) {
          const uint32_t idx = in_it + n;
          const int s = idx % kInStages;
          if (!mbar_wait(&sm.in_full[s], (idx / kInStages) & 1, kSiteFusedMma, abort)) { ok = false; break; }
          if (sdp_cnt > 0 && !mbar_wait(&sm.sdp_free, (sdp_cnt - 1) & 1, kSiteFusedMma, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.q[s]), 16, 1024);
          const uint64_t odesc = smem_desc_sw128(smem_u32(sm.dout[s]), 16, 1024);
          const uint64_t bext = smem_desc_noswizzle(smem_u32(sm.ext_b[s]), kExtLbo, kExtSbo);
          mma_ss(t_s, kdesc, qdesc, idesc_s, 0u);
#pragma unroll
          for (int kk = 1; kk < kD / 16; ++kk) mma_ss(t_s, kdesc + 2 * kk, qdesc + 2 * kk, idesc_s, 1u);
          mma_ss(t_s, aext_s, bext, idesc_s, 1u);
          mma_ss(t_dp, vdesc, odesc, idesc_s, 0u);
#pragma unroll
          for (int kk = 1; kk < kD / 16; ++kk) mma_ss(t_dp, vdesc + 2 * kk, odesc + 2 * kk, idesc_s, 1u);
          mma_ss(t_dp, aext_dp, bext, idesc_s, 1u);
          mma_commit(&sm.sdp_full);
          ++sdp_cnt;
        }
        if (!ok) break;
        in_it += n_i;
        ++it_cnt;
      }
      mma_commit(&sm.drain[0]);
      drain_wait(&sm.drain[0], 0, kSiteFusedMma);
    }
    __syncwarp();
  } else if (warp == kAccWarp) {
    // dV += P^T dO_i, dK += dS^T Q_i and dQ_ij = dS K_j once the elementwise
    // step wrote P^T (tensor memory) and dS^T (shared memory).
    if (lane == 0) {
      constexpr uint32_t idesc_tn = idesc_bf16_f32(128, 64, 0, 1);  // A K-major, B MN-major
      constexpr uint32_t idesc_nn = idesc_bf16_f32(128, 64, 1, 1);  // both MN-major
      const uint32_t t_p = tmem + 256, t_dq = tmem + 320, t_dv = tmem + 384, t_dk = tmem + 448;
      // dS^T as A: K-major for dK (K = 16 queries per step: +32 B, the second
      // 64-query half 16 KiB on); MN-major for dQ (K = 16 keys per step:
      // +2 KiB; the two 64-query halves are the M direction, 16 KiB apart).
      const uint64_t ds_k = smem_desc_sw128(smem_u32(sm.ds[0]), 16, 1024);
      const uint64_t ds_mn = smem_desc_sw128(smem_u32(sm.ds[0]), 128 * 128, 1024);
      uint32_t in_it = 0, it_cnt = 0, ds_cnt = 0, dq_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, j;
        decode(k, sh, b, h, j);
        const int slot = it_cnt & 1;
        const uint64_t kdesc_mn = smem_desc_sw128(smem_u32(sm.k[slot]), 128 * 128, 1024);
        const int n_i = n_qt - j;
        for (int n = 0; n < n_i; ++n) {
          const uint32_t idx = in_it + n;
          const int s = idx % kInStages;
          // ds_full implies this stage's Q and dO landed and S^T/dP^T are done.
          if (!mbar_wait(&sm.ds_full, ds_cnt & 1, kSiteFusedMma, abort)) { ok = false; break; }
          ++ds_cnt;
          tc_fence_after();
          const uint64_t qdesc_mn = smem_desc_sw128(smem_u32(sm.q[s]), 128 * 128, 1024);
          const uint64_t odesc_mn = smem_desc_sw128(smem_u32(sm.dout[s]), 128 * 128, 1024);
          const uint32_t acc0 = n > 0 ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < kBlockM / 16; ++kk)
            mma_ts(t_dv, t_p + 8 * kk, odesc_mn + 128 * kk, idesc_tn, kk > 0 ? 1u : acc0);
#pragma unroll
          for (int kk = 0; kk < kBlockM / 16; ++kk)
            mma_ss(t_dk, ds_k + (kk < 4 ? 2 * kk : 1024 + 2 * (kk - 4)), qdesc_mn + 128 * kk,
                   idesc_tn, kk > 0 ? 1u : acc0);
          // The dQ warps must have read the previous tile's dQ.
          if (dq_cnt > 0 && !mbar_wait(&sm.dq_free, (dq_cnt - 1) & 1, kSiteFusedMma, abort)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk)
            mma_ss(t_dq, ds_mn + 128 * kk, kdesc_mn + 128 * kk, idesc_nn, kk > 0 ? 1u : 0u);
          mma_commit(&sm.dq_full);
          ++dq_cnt;
          mma_commit(&sm.pds_free);
          mma_commit(&sm.in_empty[s]);
        }
        if (!ok) break;
        in_it += n_i;
        // Every S^T/dP^T of the item finished before its last dS^T was
        // written, and the dQ products are done: K_j and V_j are free.
        mma_commit(&sm.kv_empty[slot]);
        ++it_cnt;
      }
      mma_commit(&sm.drain[1]);
      drain_wait(&sm.drain[1], 0, kSiteFusedMma);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------- dQ sums
    const int r = ((warp & 3) << 5) + lane;  // query row within the tile = TMEM lane
    const uint32_t t_dq = tmem + (static_cast<uint32_t>((warp & 3) << 5) << 16) + 320;
    uint32_t dq_cnt = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
      const int k = snake_item(rnd, gridDim.x, blockIdx.x);
      if (k >= n_items) continue;
      int b, h, j;
      decode(k, sh, b, h, j);
      uint32_t* cnt_base = counters + (static_cast<size_t>(b) * sh.H + h) * n_qt;
      for (int i = n_qt - 1; i >= j; --i) {
        ok = mbar_wait(&sm.dq_full, dq_cnt & 1, kSiteFusedSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++dq_cnt;
        tc_fence_after();
        uint32_t q[64];
        tmem_ld32(t_dq, *reinterpret_cast<uint32_t(*)[32]>(q));
        tmem_ld32(t_dq + 32, *reinterpret_cast<uint32_t(*)[32]>(q + 32));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.dq_free);
        ok = add_dq(q, dq_sum, cnt_base + i, dqkv, b, h, i, j, r, lane, n_qt, C, sh, abort);
        if (!ok) break;
      }
      if (!ok) break;
      // Release the item's query tiles above the diagonal (the diagonal one
      // was the last contributor and is final): this warp's sums are visible
      // before any count says so.
      __syncwarp();
      if (lane == 0 && j < n_qt - 1) {
        fence_acq_rel_gpu();
        for (int i = j + 1; i < n_qt; ++i) atomicAdd(cnt_base + i, 1u);
      }
    }
  } else {
    // ------------------------------------------------------- elementwise WGs
    const int r = ((warp & 3) << 5) + lane;  // key row within the tile = TMEM lane
    const int g = warp >> 2;                 // query columns [32g, 32g + 32)
    const int r_lo = (warp & 3) << 5;
    const uint32_t lb = static_cast<uint32_t>(r_lo) << 16;
    const uint32_t t_s = tmem + lb + 32 * g, t_dp = tmem + lb + 128 + 32 * g;
    const uint32_t t_p = tmem + lb + 256 + 16 * g;
    const uint32_t t_dv = tmem + lb + 384 + 16 * g, t_dk = tmem + lb + 448 + 16 * g;
    const float sc = sh.scale_log2;
    uint32_t sdp_cnt = 0, pds_cnt = 0, tiles = 0;
    // The finished item whose dV, dK still sit in tensor memory (read out
    // during the next item's first tile).
    bool pending = false;
    int pb = 0, ph = 0, pj = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
      const int k = snake_item(rnd, gridDim.x, blockIdx.x);
      if (k >= n_items) continue;
      int b, h, j;
      decode(k, sh, b, h, j);
      for (int i = n_qt - 1; i >= j; --i, ++tiles) {
        ok = mbar_wait(&sm.sdp_full, sdp_cnt & 1, kSiteFusedSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sdp_cnt;
        tc_fence_after();
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sv[16], dv[16];
          tmem_ld16(t_s + 16 * half, sv);
          tmem_ld16(t_dp + 16 * half, dv);
          tmem_wait_ld();
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sdp_free);
          }
          const int c0 = 32 * g + 16 * half;  // first query column of the chunk
          uint32_t (&pph)[8] = *reinterpret_cast<uint32_t(*)[8]>(pp + 8 * half);
          uint32_t (&ddh)[8] = *reinterpret_cast<uint32_t(*)[8]>(dd + 8 * half);
          if (i == j && c0 < r_lo + 31)
            dkdv_chunk<true>(sv, dv, sc, c0, r, pph, ddh);
          else
            dkdv_chunk<false>(sv, dv, sc, c0, r, pph, ddh);
        }
        const bool have_prev = tiles > 0;
        const bool flush = (i == n_qt - 1) && pending;
        if (have_prev) {
          // The previous tile's dV/dK/dQ products are done: P^T and dS^T may
          // be reused.
          ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteFusedSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++pds_cnt;
          tc_fence_after();
          if (flush) {
            uint32_t av[16], ak[16];
            tmem_ld16(t_dv, av);
            tmem_ld16(t_dk, ak);
            tmem_wait_ld();
            store_dkdv_row(dqkv, av, ak, pb, ph, pj, r, g, C, sh);
            pending = false;
          }
        }
        tmem_st16(t_p, pp);
        store_ds_row(sm, dd, r, g);
        fence_proxy_async_smem();  // generic-proxy dS^T stores -> tensor core
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
      }
      if (!ok) break;
      pending = true;
      pb = b;
      ph = h;
      pj = j;
    }
    if (ok && tiles > 0) {
      ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteFusedSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        ++pds_cnt;
        tc_fence_after();
        uint32_t av[16], ak[16];
        tmem_ld16(t_dv, av);
        tmem_ld16(t_dk, ak);
        tmem_wait_ld();
        tc_fence_before();
        store_dkdv_row(dqkv, av, ak, pb, ph, pj, r, g, C, sh);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fused
}  // namespace bwd
}  // namespace ga
