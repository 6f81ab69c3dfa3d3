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
// Two kernels, launched in this order on one stream:
//   attn_bwd_dq_kernel   one CTA per 128-query tile i: computes the tile's
//                        Delta from its dO and O tiles (and writes it out),
//                        streams key tiles j <= i, accumulates dQ in tensor
//                        memory.
//   attn_bwd_dkdv_kernel one CTA per 128-key tile j: streams query tiles
//                        i >= j (reading Delta), accumulates dK and dV in
//                        tensor memory.
// Nothing is accumulated through atomics, so the result is bitwise
// deterministic. attn_bwd_pre_kernel computes Delta on its own, for callers
// of the separate preprocessing step and for the fused backward.
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
// Also zeroes `n_counters` words at `counters` (the fused backward's dQ
// ordering counters; none for the split backward).
__global__ void __launch_bounds__(256)
attn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                    float* __restrict__ delta, uint32_t* __restrict__ counters, int n_counters,
                    const AttnShape sh) {
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < n_counters; c += gridDim.x * blockDim.x)
    counters[c] = 0u;
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
// Warps 0-15: four elementwise warpgroups. Each thread owns one row of the
// tile (its TMEM lane); warpgroup g takes the 32 columns [32g, 32g + 32).
// Warp 16: TMA producer. Warp 17: issues the S and dP products (and owns the
// tensor-memory allocation). Warp 18: issues the accumulating products (dV and
// dK, or dQ). Two issuing threads let the next tile's S/dP enter the tensor
// pipe while the current tile's accumulation waits for its elementwise step.
constexpr int kThreads = 608;
constexpr int kEwWarps = 16;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kAccWarp = 18;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ===========================================================================
// dK, dV: one CTA per key tile
// ===========================================================================
// Per query tile i >= j (all in the transposed frame, rows = keys):
//   S'^T  = K_j Q_i^T - lse_i/scale   (M128 N128, K = 64 + one extra K16 step)
//   dP'^T = V_j dO_i^T - Delta_i      (same)
//   P^T   = exp2(S'^T * scale*log2e), zero where key > query
//   dS^T  = P^T o dP'^T
// The extra K step multiplies a constant tile A_ext (rows of ones in the
// columns that pick a term) with a per-query tile B_ext holding -lse/scale and
// -Delta, each split into three bf16 terms whose sum is exact to ~2^-24
// relative. The per-query constants thus never pass through the elementwise
// warps, which would otherwise broadcast them from shared memory while the
// S/dP products saturate it.
//   dV  += P^T dO_i      (A = P^T from tensor memory, B = dO_i MN-major)
//   dK  += dS^T Q_i      (A = dS^T from tensor memory, B = Q_i MN-major)
// Tensor memory: S^T [0,128), dP^T [128,256), P^T [256,320), dS^T [320,384)
// (bf16 pairs), dV [384,448), dK [448,512).
// 16 columns of one dK/dV tile row. The accumulators already hold
// S^T - lse/scale and dP^T - Delta (one extra K step of each product adds the
// per-query constants), so P^T = 2^(c x) (zero where the key r comes after
// query c0 + e when kMasked) and dS^T = P^T o dP'^T, both packed to bf16 pairs.
template <bool kMasked>
__device__ __forceinline__ void dkdv_chunk(const uint32_t (&sv)[16], const uint32_t (&dv)[16],
                                           float sc, int c0, int r, uint32_t (&pp)[8],
                                           uint32_t (&dd)[8]) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    float x0, x1, d0, d1;
    mul2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sc, x0, x1);
    if (kMasked) {
      if (c0 + c < r) x0 = -INFINITY;
      if (c0 + c + 1 < r) x1 = -INFINITY;
    }
    const float p0 = ex2(x0), p1 = ex2(x1);
    mul2v(p0, p1, __uint_as_float(dv[c]), __uint_as_float(dv[c + 1]), d0, d1);
    pp[c >> 1] = pack_bf16(p0, p1);
    dd[c >> 1] = pack_bf16(d0, d1);
  }
}

// 16 columns of one dQ tile row: P = 2^(S c - lse c) (zero where key
// c0 + e comes after the query r when kMasked), dS = P (dP - Delta) as bf16
// pairs. nl = -lse*log2(e) and nd = -Delta of the row.
template <bool kMasked>
__device__ __forceinline__ void dq_chunk(const uint32_t (&sv)[16], const uint32_t (&dv)[16],
                                         float nl, float nd, float sc, int c0, int r,
                                         uint32_t (&dd)[8]) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    float x0, x1, d0, d1;
    fma2v(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1]), sc, sc, nl, nl, x0, x1);
    if (kMasked) {
      if (c0 + c > r) x0 = -INFINITY;
      if (c0 + c + 1 > r) x1 = -INFINITY;
    }
    const float p0 = ex2(x0), p1 = ex2(x1);
    float t0 = __uint_as_float(dv[c]), t1 = __uint_as_float(dv[c + 1]);
    add2(t0, t1, nd, nd);
    mul2v(p0, p1, t0, t1, d0, d1);
    dd[c >> 1] = pack_bf16(d0, d1);
  }
}

// Stores one key row of dV (slot 2) and dK * scale (slot 1): warpgroup g
// writes d columns [16g, 16g + 16) from its fp32 accumulator values.
__device__ __forceinline__ void store_dkdv_row(__nv_bfloat16* dqkv, const uint32_t (&av)[16],
                                               const uint32_t (&ak)[16], int b, int h, int j,
                                               int r, int g, int C, const AttnShape& sh) {
  const int key = j * kBlockN + r;
  if (key >= sh.T) return;
  __nv_bfloat16* base = dqkv + ((static_cast<size_t>(b) * sh.T + key) * 3) * C + h * kD + 16 * g;
  uint4* dst_v = reinterpret_cast<uint4*>(base + 2 * C);
  uint4* dst_k = reinterpret_cast<uint4*>(base + C);
  const float s = sh.scale;
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    dst_v[v] = make_uint4(pack_bf16(__uint_as_float(av[8 * v]), __uint_as_float(av[8 * v + 1])),
                          pack_bf16(__uint_as_float(av[8 * v + 2]), __uint_as_float(av[8 * v + 3])),
                          pack_bf16(__uint_as_float(av[8 * v + 4]), __uint_as_float(av[8 * v + 5])),
                          pack_bf16(__uint_as_float(av[8 * v + 6]), __uint_as_float(av[8 * v + 7])));
    dst_k[v] = make_uint4(pack_bf16(__uint_as_float(ak[8 * v]) * s, __uint_as_float(ak[8 * v + 1]) * s),
                          pack_bf16(__uint_as_float(ak[8 * v + 2]) * s, __uint_as_float(ak[8 * v + 3]) * s),
                          pack_bf16(__uint_as_float(ak[8 * v + 4]) * s, __uint_as_float(ak[8 * v + 5]) * s),
                          pack_bf16(__uint_as_float(ak[8 * v + 6]) * s, __uint_as_float(ak[8 * v + 7]) * s));
  }
}

// Stores one query row of dQ * scale (slot 0), d columns [16g, 16g + 16).
__device__ __forceinline__ void store_dq_row(__nv_bfloat16* dqkv, const uint32_t (&aq)[16], int b,
                                             int h, int row, int g, int C, const AttnShape& sh) {
  if (row >= sh.T) return;
  const float s = sh.scale;
  uint4* dst =
      reinterpret_cast<uint4*>(dqkv + ((static_cast<size_t>(b) * sh.T + row) * 3) * C + h * kD + 16 * g);
#pragma unroll
  for (int v = 0; v < 2; ++v)
    dst[v] = make_uint4(pack_bf16(__uint_as_float(aq[8 * v]) * s, __uint_as_float(aq[8 * v + 1]) * s),
                        pack_bf16(__uint_as_float(aq[8 * v + 2]) * s, __uint_as_float(aq[8 * v + 3]) * s),
                        pack_bf16(__uint_as_float(aq[8 * v + 4]) * s, __uint_as_float(aq[8 * v + 5]) * s),
                        pack_bf16(__uint_as_float(aq[8 * v + 6]) * s, __uint_as_float(aq[8 * v + 7]) * s));
}

namespace dkdv {

constexpr uint32_t kExtBytes = 128 * 32;  // 128 rows x 16 bf16 (one K16 step)
constexpr uint32_t kExtLbo = 128, kExtSbo = 256;

// Byte offset of row `r`'s first 8 terms in an A_ext / B_ext tile.
__device__ __forceinline__ uint32_t ext_row(int r) { return (r >> 3) * kExtSbo + (r & 7) * 16; }

// v as three bf16 terms, each the nearest bf16 of what the previous ones
// leave over: |v - (h1 + h2 + h3)| <= 2^-24 |v| (up to subnormals).
__device__ __forceinline__ void split3_bf16(float v, __nv_bfloat16& h1, __nv_bfloat16& h2,
                                            __nv_bfloat16& h3) {
  h1 = __float2bfloat16_rn(v);
  const float r1 = v - __bfloat162float(h1);
  h2 = __float2bfloat16_rn(r1);
  h3 = __float2bfloat16_rn(r1 - __bfloat162float(h2));
}

__device__ __forceinline__ uint32_t bf16_pair(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

struct alignas(1024) Smem {
  // [item slot] K_j and V_j of the item; once the item's last products have
  // read them, the same bytes stage its dK and dV tiles (bf16, 128-byte
  // swizzle) on their way to global memory.
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  uint8_t q[kStages][kTileBytes];
  uint8_t dout[kStages][kTileBytes];
  // K-major, no swizzle: 8-row x 16-byte core matrices, 128 bytes apart along K
  // (two per K16 step) and 256 bytes apart along the rows.
  uint8_t ext_a[2][kExtBytes];        // [S, dP]: ones in terms 0-2 / 3-5 of every key row
  uint8_t ext_b[kStages][kExtBytes];  // per query row: 3 terms of -lse/scale, 3 of -Delta
  uint64_t kv_full[2], kv_empty[2];
  uint64_t in_full[kStages], in_empty[kStages];
  uint64_t sdp_full, sdp_free, ds_full, pds_free;
  uint64_t ostage_full;  // the finished item's dK/dV rows are staged
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "dK/dV shared memory exceeds the 227 KiB per-block limit");

// Row r's 16 columns [16g, 16g + 16) of dV and of dK * scale, as bf16, into
// the staging tiles (128-byte swizzle: 16-byte chunk c of row r at
// r * 128 + ((c ^ (r & 7)) << 4)); chunks 2g and 2g + 1.
__device__ __forceinline__ void stage_dkdv_row(uint8_t* dk_tile, uint8_t* dv_tile,
                                               const uint32_t (&av)[16], const uint32_t (&ak)[16],
                                               int r, int g, float s) {
#pragma unroll
  for (int v = 0; v < 2; ++v) {
    const int off = r * 128 + (((2 * g + v) ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(dv_tile + off) =
        make_uint4(pack_bf16(__uint_as_float(av[8 * v]), __uint_as_float(av[8 * v + 1])),
                   pack_bf16(__uint_as_float(av[8 * v + 2]), __uint_as_float(av[8 * v + 3])),
                   pack_bf16(__uint_as_float(av[8 * v + 4]), __uint_as_float(av[8 * v + 5])),
                   pack_bf16(__uint_as_float(av[8 * v + 6]), __uint_as_float(av[8 * v + 7])));
    *reinterpret_cast<uint4*>(dk_tile + off) =
        make_uint4(pack_bf16(__uint_as_float(ak[8 * v]) * s, __uint_as_float(ak[8 * v + 1]) * s),
                   pack_bf16(__uint_as_float(ak[8 * v + 2]) * s, __uint_as_float(ak[8 * v + 3]) * s),
                   pack_bf16(__uint_as_float(ak[8 * v + 4]) * s, __uint_as_float(ak[8 * v + 5]) * s),
                   pack_bf16(__uint_as_float(ak[8 * v + 6]) * s, __uint_as_float(ak[8 * v + 7]) * s));
  }
}

__device__ __forceinline__ void decode(int k, const AttnShape& sh, int& b, int& h, int& j) {
  const int bh_count = sh.B * sh.H;
  j = k / bh_count;  // key tile 0 has the most query tiles: heaviest first
  const int bh = k % bh_count;
  b = bh / sh.H;
  h = bh % sh.H;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_qkv,
                     const __grid_constant__ CUtensorMap map_do,
                     const __grid_constant__ CUtensorMap map_dqkv, const float* __restrict__ lse,
                     const float* __restrict__ delta, const AttnShape sh) {
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
      // The item's last products (commit) and the store of its dK/dV tiles
      // out of the same bytes (lane 0 of warp 0, once the bulk stores have
      // read them).
      mbar_init(&sm.kv_empty[s], 2);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.in_full[s], 2);  // TMA bytes + the warp's lse/Delta stores
      mbar_init(&sm.in_empty[s], 1);
    }
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.sdp_free, kEwWarps);
    mbar_init(&sm.ds_full, kEwWarps);
    mbar_init(&sm.pds_free, 1);
    mbar_init(&sm.ostage_full, kEwWarps);
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  // A_ext rows pick terms 0-2 (S) or 3-5 (dP) of B_ext; B_ext's second core
  // matrix along K (terms 8-15) stays zero. Written through the generic proxy,
  // so every writer fences before the tensor core may read them.
  for (int idx = threadIdx.x; idx < 2 * kBlockN; idx += kThreads) {
    const int which = idx / kBlockN, rr = idx % kBlockN;
    uint4* a = reinterpret_cast<uint4*>(sm.ext_a[which] + ext_row(rr));
    a[0] = which == 0 ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u)
                      : make_uint4(0u, 0x3F800000u, 0x3F803F80u, 0u);
    a[kExtLbo / 16] = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int idx = threadIdx.x; idx < kStages * static_cast<int>(kExtBytes / 16); idx += kThreads)
    reinterpret_cast<uint4*>(&sm.ext_b[0][0])[idx] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_qkv);
    tma_prefetch_desc(&map_do);
    tma_prefetch_desc(&map_dqkv);
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
      for (int s = 0; s < kStages; ++s)
        if (in_it > static_cast<uint32_t>(s))
          drain_wait(&sm.in_full[s], ((in_it - s + kStages - 1) / kStages - 1) & 1, kSiteDkvProducer);
      for (int s = 0; s < 2; ++s)
        if (it_cnt > static_cast<uint32_t>(s))
          drain_wait(&sm.kv_full[s], ((it_cnt - s + 1) / 2 - 1) & 1, kSiteDkvProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // S'^T and dP'^T (with the extra K step) for every query tile i >= j.
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
        if (!mbar_wait(&sm.kv_full[slot], (it_cnt >> 1) & 1, kSiteDkvMma, abort)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[slot]), 16, 1024);
        const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[slot]), 16, 1024);
        const int n_i = n_qt - j;
        for (int n = 0; n < n_i; ++n) {
          const uint32_t idx = in_it + n;
          const int s = idx % kStages;
          if (!mbar_wait(&sm.in_full[s], (idx / kStages) & 1, kSiteDkvMma, abort)) { ok = false; break; }
          if (sdp_cnt > 0 && !mbar_wait(&sm.sdp_free, (sdp_cnt - 1) & 1, kSiteDkvMma, abort)) { ok = false; break; }
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
      drain_wait(&sm.drain[0], 0, kSiteDkvMma);
    }
    __syncwarp();
  } else if (warp == kAccWarp) {
    // dV += P^T dO_i and dK += dS^T Q_i once the elementwise step wrote them.
    if (lane == 0) {
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t t_p = tmem + 256, t_ds = tmem + 320, t_dv = tmem + 384, t_dk = tmem + 448;
      uint32_t in_it = 0, it_cnt = 0, ds_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, j;
        decode(k, sh, b, h, j);
        const int slot = it_cnt & 1;
        const int n_i = n_qt - j;
        for (int n = 0; n < n_i; ++n) {
          const uint32_t idx = in_it + n;
          const int s = idx % kStages;
          // ds_full implies this stage's Q and dO landed and S^T/dP^T are done.
          if (!mbar_wait(&sm.ds_full, ds_cnt & 1, kSiteDkvMma, abort)) { ok = false; break; }
          ++ds_cnt;
          tc_fence_after();
          const uint64_t qdesc_mn = smem_desc_sw128(smem_u32(sm.q[s]), 128 * 128, 1024);
          const uint64_t odesc_mn = smem_desc_sw128(smem_u32(sm.dout[s]), 128 * 128, 1024);
          const uint32_t acc0 = n > 0 ? 1u : 0u;
          mma_ts(t_dv, t_p, odesc_mn, idesc_acc, acc0);
#pragma unroll
          for (int kk = 1; kk < kBlockM / 16; ++kk)
            mma_ts(t_dv, t_p + 8 * kk, odesc_mn + 128 * kk, idesc_acc, 1u);
          mma_ts(t_dk, t_ds, qdesc_mn, idesc_acc, acc0);
#pragma unroll
          for (int kk = 1; kk < kBlockM / 16; ++kk)
            mma_ts(t_dk, t_ds + 8 * kk, qdesc_mn + 128 * kk, idesc_acc, 1u);
          mma_commit(&sm.pds_free);
          mma_commit(&sm.in_empty[s]);
        }
        if (!ok) break;
        in_it += n_i;
        // Every S^T/dP^T of the item finished before its last dS^T was written,
        // so this also releases K_j and V_j.
        mma_commit(&sm.kv_empty[slot]);
        ++it_cnt;
      }
      mma_commit(&sm.drain[1]);
      drain_wait(&sm.drain[1], 0, kSiteDkvMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- elementwise WGs
    const int r = ((warp & 3) << 5) + lane;  // key row within the tile = TMEM lane
    const int g = warp >> 2;                 // query columns [32g, 32g + 32)
    const int r_lo = (warp & 3) << 5;        // first row of this warp
    const uint32_t lb = static_cast<uint32_t>(r_lo) << 16;
    const uint32_t t_s = tmem + lb + 32 * g, t_dp = tmem + lb + 128 + 32 * g;
    const uint32_t t_p = tmem + lb + 256 + 16 * g, t_ds = tmem + lb + 320 + 16 * g;
    const uint32_t t_dv = tmem + lb + 384 + 16 * g, t_dk = tmem + lb + 448 + 16 * g;
    const float sc = sh.scale_log2;
    uint32_t sdp_cnt = 0, pds_cnt = 0, in_it = 0, ost_cnt = 0;
    // The finished item's dK and dV rows go to global memory through the
    // item's own K and V tiles (slot `ps`), which its last products have
    // finished reading (the item's last dV/dK product completed before this
    // warp read the accumulators): every warp writes its rows there, and lane
    // 0 of warp 0 stores both 128 x 64 tiles with two TMA bulk stores (dqkv
    // slots 1 and 2; rows past T are clipped), then releases the slot to the
    // loads of the item after next. Scattered 32-byte stores from every
    // thread, one segment per row, held all 16 warps for ~2000 cycles per
    // item. Returns false if a wait gave up.
    auto emit_dkdv = [&](const uint32_t (&av)[16], const uint32_t (&ak)[16], int eb, int eh,
                         int ej, int ps) -> bool {
      stage_dkdv_row(sm.k[ps], sm.v[ps], av, ak, r, g, sh.scale);
      fence_proxy_async_smem();  // generic-proxy writes, read by the TMA engine
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.ostage_full);
      bool w = true;
      if (warp == 0 && lane == 0) {
        w = mbar_wait(&sm.ostage_full, ost_cnt & 1, kSiteDkvSoftmax, abort);
        if (w) {
          tma_store_3d(&map_dqkv, sm.k[ps], C + eh * kD, ej * kBlockN, eb);
          tma_store_3d(&map_dqkv, sm.v[ps], 2 * C + eh * kD, ej * kBlockN, eb);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(&sm.kv_empty[ps]);
        }
      }
      ++ost_cnt;
      return __all_sync(0xffffffffu, w);
    };
    int item_cnt = 0, ps = 0;
    // The finished item whose dV, dK still sit in tensor memory: they are read
    // out while the next item's first tile is processed, just before its P^T
    // and dS^T go to tensor memory (after which the next dV/dK product
    // overwrites the accumulators).
    bool pending = false;
    int pb = 0, ph = 0, pj = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
      const int k = snake_item(rnd, gridDim.x, blockIdx.x);
      if (k >= n_items) continue;
      int b, h, j;
      decode(k, sh, b, h, j);
      for (int i = j; i < n_qt; ++i, ++in_it) {
        ok = mbar_wait(&sm.sdp_full, sdp_cnt & 1, kSiteDkvSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sdp_cnt;
        tc_fence_after();
        // Both 16-column halves are computed into registers before waiting for
        // the previous dV/dK products to release P^T and dS^T, so that wait
        // overlaps all of this tile's elementwise work.
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
          // On the diagonal tile, a chunk needs the mask if one of its columns
          // lies before one of this warp's rows (key after query).
          if (i == j && c0 < r_lo + 31)
            dkdv_chunk<true>(sv, dv, sc, c0, r, pph, ddh);
          else
            dkdv_chunk<false>(sv, dv, sc, c0, r, pph, ddh);
        }
        const bool flush = (i == j) && pending;
        if (i > j || flush) {
          // The previous dV/dK products must be done reading P^T and dS^T; on
          // an item's first tile that is the finished item's last product.
          ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteDkvSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++pds_cnt;
          tc_fence_after();
        }
        if (flush) {
          // Read the finished item's accumulators out before this tile's dV/dK
          // product overwrites them; store them once this tile is handed over.
          uint32_t av[16], ak[16];
          tmem_ld16(t_dv, av);
          tmem_ld16(t_dk, ak);
          tmem_wait_ld();
          tmem_st16(t_p, pp);
          tmem_st16(t_ds, dd);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.ds_full);
          ok = emit_dkdv(av, ak, pb, ph, pj, ps);
          if (!ok) break;
          pending = false;
        } else {
          tmem_st16(t_p, pp);
          tmem_st16(t_ds, dd);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.ds_full);
        }
      }
      if (!ok) break;
      pending = true;
      pb = b;
      ph = h;
      pj = j;
      ps = item_cnt & 1;
      ++item_cnt;
    }
    if (ok && pending) {
      ok = mbar_wait(&sm.pds_free, pds_cnt & 1, kSiteDkvSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        ++pds_cnt;
        tc_fence_after();
        uint32_t av[16], ak[16];
        tmem_ld16(t_dv, av);
        tmem_ld16(t_dk, ak);
        tmem_wait_ld();
        tc_fence_before();
        emit_dkdv(av, ak, pb, ph, pj, ps);
      }
    }
    // Every bulk store this CTA issued has completed before it exits.
    if (warp == 0 && lane == 0) bulk_wait_group0();
    __syncwarp();
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
  uint8_t o[2][kTileBytes];  // the forward's output tile, for Delta
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t in_full[2], in_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t sdp_full, sdp_free, ds_full, acc_done;
  uint64_t ds_free[2];  // dS buffer b no longer read by a dQ product
  uint64_t drain[2];
  uint64_t dpart_full[2];  // [item slot] the four Delta partial sums are in place
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 232448, "dQ shared memory exceeds the 227 KiB per-block limit");

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ int sw128_chunk(int r, int c) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

// Column group g's share of Delta for query row r: sum over columns
// [16g, 16g + 16) of dO[r][d] * O[r][d] (chunks 2g and 2g + 1 of each row).
// Only this thread reads those O bytes, so it then leaves the partial sum in
// the first word of its chunk 2g, where the other groups pick it up.
__device__ __forceinline__ void delta_part(const uint8_t* dout_tile, uint8_t* o_tile, int r,
                                           int g) {
  const int off0 = sw128_chunk(r, 2 * g), off1 = sw128_chunk(r, 2 * g + 1);
  const uint4 a0 = *reinterpret_cast<const uint4*>(dout_tile + off0);
  const uint4 a1 = *reinterpret_cast<const uint4*>(dout_tile + off1);
  const uint4 o0 = *reinterpret_cast<const uint4*>(o_tile + off0);
  const uint4 o1 = *reinterpret_cast<const uint4*>(o_tile + off1);
  const uint32_t ua[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const uint32_t uo[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc[e & 3] = fmaf(__uint_as_float(ua[e] << 16), __uint_as_float(uo[e] << 16), acc[e & 3]);
    acc[e & 3] = fmaf(__uint_as_float(ua[e] & 0xFFFF0000u), __uint_as_float(uo[e] & 0xFFFF0000u),
                      acc[e & 3]);
  }
  *reinterpret_cast<float*>(o_tile + off0) = (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Delta of row r: the four groups' partial sums, added in one fixed order.
__device__ __forceinline__ float delta_sum(const uint8_t* o_tile, int r) {
  const float p0 = *reinterpret_cast<const float*>(o_tile + sw128_chunk(r, 0));
  const float p1 = *reinterpret_cast<const float*>(o_tile + sw128_chunk(r, 2));
  const float p2 = *reinterpret_cast<const float*>(o_tile + sw128_chunk(r, 4));
  const float p3 = *reinterpret_cast<const float*>(o_tile + sw128_chunk(r, 6));
  return (p0 + p1) + (p2 + p3);
}

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
                   const __grid_constant__ CUtensorMap map_do,
                   const __grid_constant__ CUtensorMap map_o, const float* __restrict__ lse,
                   float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv,
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
    for (int d = 0; d < 2; ++d) {
      mbar_init(&sm.ds_free[d], 1);
      mbar_init(&sm.drain[d], 1);
      mbar_init(&sm.dpart_full[d], kEwWarps);
    }
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_qkv);
    tma_prefetch_desc(&map_do);
    tma_prefetch_desc(&map_o);
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
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, i;
        decode(k, sh, n_qt, b, h, i);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.in_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteDqProducer, abort)) break;
        mbar_arrive_expect_tx(&sm.in_full[slot], 3 * kTileBytes);
        tma_load_3d(sm.q[slot], &map_qkv, &sm.in_full[slot], h * kD, i * kBlockM, b);
        tma_load_3d(sm.dout[slot], &map_do, &sm.in_full[slot], h * kD, i * kBlockM, b);
        tma_load_3d(sm.o[slot], &map_o, &sm.in_full[slot], h * kD, i * kBlockM, b);
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
    // S = Q_i K_j^T and dP = dO_i V_j^T for every key tile j <= i.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t t_s = tmem + 0, t_dp = tmem + 128;
      uint32_t kv_it = 0, it_cnt = 0, sdp_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, i;
        decode(k, sh, n_qt, b, h, i);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.in_full[slot], (it_cnt >> 1) & 1, kSiteDqMma, abort)) { ok = false; break; }
        tc_fence_after();
        const uint64_t qdesc = smem_desc_sw128(smem_u32(sm.q[slot]), 16, 1024);
        const uint64_t odesc = smem_desc_sw128(smem_u32(sm.dout[slot]), 16, 1024);
        const int n_j = i + 1;
        for (int n = 0; n < n_j; ++n) {
          const uint32_t idx = kv_it + n;
          const int s = idx % kStages;
          if (!mbar_wait(&sm.kv_full[s], (idx / kStages) & 1, kSiteDqMma, abort)) { ok = false; break; }
          if (sdp_cnt > 0 && !mbar_wait(&sm.sdp_free, (sdp_cnt - 1) & 1, kSiteDqMma, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[s]), 16, 1024);
          const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[s]), 16, 1024);
          mma_ss(t_s, qdesc, kdesc, idesc_s, 0u);
#pragma unroll
          for (int kk = 1; kk < kD / 16; ++kk) mma_ss(t_s, qdesc + 2 * kk, kdesc + 2 * kk, idesc_s, 1u);
          mma_ss(t_dp, odesc, vdesc, idesc_s, 0u);
#pragma unroll
          for (int kk = 1; kk < kD / 16; ++kk) mma_ss(t_dp, odesc + 2 * kk, vdesc + 2 * kk, idesc_s, 1u);
          mma_commit(&sm.sdp_full);
          ++sdp_cnt;
        }
        if (!ok) break;
        kv_it += n_j;
        ++it_cnt;
      }
      mma_commit(&sm.drain[0]);
      drain_wait(&sm.drain[0], 0, kSiteDqMma);
    }
    __syncwarp();
  } else if (warp == kAccWarp) {
    // dQ += dS K_j once the elementwise step wrote dS.
    if (lane == 0) {
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t t_ds0 = tmem + 256, t_dq = tmem + 384;
      uint32_t kv_it = 0, it_cnt = 0, ds_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
        const int k = snake_item(rnd, gridDim.x, blockIdx.x);
        if (k >= n_items) continue;
        int b, h, i;
        decode(k, sh, n_qt, b, h, i);
        const int slot = it_cnt & 1;
        const int n_j = i + 1;
        for (int n = 0; n < n_j; ++n) {
          const uint32_t idx = kv_it + n;
          const int s = idx % kStages;
          // ds_full implies this stage's K landed and S/dP are done.
          if (!mbar_wait(&sm.ds_full, ds_cnt & 1, kSiteDqMma, abort)) { ok = false; break; }
          const int buf = ds_cnt & 1;
          const uint32_t t_ds = t_ds0 + 64 * buf;
          ++ds_cnt;
          tc_fence_after();
          const uint64_t kdesc_mn = smem_desc_sw128(smem_u32(sm.k[s]), 128 * 128, 1024);
          mma_ts(t_dq, t_ds, kdesc_mn, idesc_acc, n > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < kBlockN / 16; ++kk)
            mma_ts(t_dq, t_ds + 8 * kk, kdesc_mn + 128 * kk, idesc_acc, 1u);
          mma_commit(&sm.ds_free[buf]);
          // S/dP of this key tile finished before its dS was written, so the
          // stage can be refilled once this product is done.
          mma_commit(&sm.kv_empty[s]);
        }
        if (!ok) break;
        kv_it += n_j;
        mma_commit(&sm.acc_done);
        mma_commit(&sm.in_empty[slot]);
        ++it_cnt;
      }
      mma_commit(&sm.drain[1]);
      drain_wait(&sm.drain[1], 0, kSiteDqMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------- elementwise WGs
    const int r = ((warp & 3) << 5) + lane;  // query row within the tile = TMEM lane
    const int g = warp >> 2;                 // key columns [32g, 32g + 32)
    const int r_lo = (warp & 3) << 5;
    const uint32_t lb = static_cast<uint32_t>(r_lo) << 16;
    const uint32_t t_s = tmem + lb + 32 * g, t_dp = tmem + lb + 128 + 32 * g;
    const uint32_t t_ds0 = tmem + lb + 256 + 16 * g, t_dq = tmem + lb + 384 + 16 * g;
    const float sc = sh.scale_log2;
    uint32_t sdp_cnt = 0, acc_cnt = 0, ds_cnt = 0, it_cnt = 0;
    // The finished item whose dQ still sits in tensor memory: it is read out
    // while the next item's first tile is processed, just before that tile's
    // dS goes to tensor memory (after which the next dQ product overwrites
    // the accumulator).
    bool pending = false;
    int pb = 0, ph = 0, prow = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd * static_cast<int>(gridDim.x) < n_items; ++rnd) {
      const int k = snake_item(rnd, gridDim.x, blockIdx.x);
      if (k >= n_items) continue;
      int b, h, i;
      decode(k, sh, n_qt, b, h, i);
      const int row = i * kBlockM + r;
      const bool valid = row < sh.T;
      const size_t lrow = (static_cast<size_t>(b) * sh.H + h) * sh.T + row;
      // Rows past T get -lse = -inf (P = 0).
      const float nl = valid ? -lse[lrow] * kLog2e : -INFINITY;
      // Delta of this row from the item's dO and O tiles (their in_full phase
      // makes the TMA writes visible here): each column group sums a quarter
      // of the columns, the partial sums meet in the O tile (which nothing
      // else reads), and every group adds the four in the same order. The
      // first group writes Delta out for the dK/dV kernel. The O slot is
      // reloaded only after this item's last dQ product, long after these
      // reads.
      const int slot = it_cnt & 1;
      const uint32_t item_parity = (it_cnt >> 1) & 1;
      ok = mbar_wait(&sm.in_full[slot], item_parity, kSiteDqSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      delta_part(sm.dout[slot], sm.o[slot], r, g);
      fence_proxy_async_smem();  // order these writes before the slot's next TMA load
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.dpart_full[slot]);
      ok = mbar_wait(&sm.dpart_full[slot], item_parity, kSiteDqSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++it_cnt;
      const float dl = delta_sum(sm.o[slot], r);
      if (valid && g == 0) delta[lrow] = dl;
      const float nd = valid ? -dl : 0.f;
      for (int j = 0; j <= i; ++j) {
        ok = mbar_wait(&sm.sdp_full, sdp_cnt & 1, kSiteDqSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++sdp_cnt;
        tc_fence_after();
        const int buf = ds_cnt & 1;
        const uint32_t t_ds = t_ds0 + 64 * buf;
        const uint32_t uses = ds_cnt >> 1;  // earlier dS tiles written to this buffer
        ++ds_cnt;
        uint32_t dd[16];
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // 16 key columns at a time
          uint32_t sv[16], dv[16];
          tmem_ld16(t_s + 16 * half, sv);
          tmem_ld16(t_dp + 16 * half, dv);
          tmem_wait_ld();
          if (half == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sdp_free);
          }
          const int c0 = 32 * g + 16 * half;  // first key column of the chunk
          uint32_t (&ddh)[8] = *reinterpret_cast<uint32_t(*)[8]>(dd + 8 * half);
          // On the diagonal tile, a chunk needs the mask if one of its keys lies
          // after one of this warp's queries.
          if (j == i && c0 + 15 > r_lo)
            dq_chunk<true>(sv, dv, nl, nd, sc, c0, r, ddh);
          else
            dq_chunk<false>(sv, dv, nl, nd, sc, c0, r, ddh);
        }
        if (uses > 0) {
          // The dQ product that read this buffer two tiles ago must be done.
          ok = mbar_wait(&sm.ds_free[buf], (uses - 1) & 1, kSiteDqSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
        if (j == 0 && pending) {
          // Read the finished item's dQ out before this tile's dQ product
          // overwrites it; store it once this tile is handed over.
          ok = mbar_wait(&sm.acc_done, acc_cnt & 1, kSiteDqSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++acc_cnt;
          tc_fence_after();
          uint32_t aq[16];
          tmem_ld16(t_dq, aq);
          tmem_wait_ld();
          tmem_st16(t_ds, dd);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.ds_full);
          store_dq_row(dqkv, aq, pb, ph, prow, g, C, sh);
          pending = false;
        } else {
          tmem_st16(t_ds, dd);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.ds_full);
        }
      }
      if (!ok) break;
      pending = true;
      pb = b;
      ph = h;
      prow = row;
    }
    if (ok && pending) {
      ok = mbar_wait(&sm.acc_done, acc_cnt & 1, kSiteDqSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        ++acc_cnt;
        tc_fence_after();
        uint32_t aq[16];
        tmem_ld16(t_dq, aq);
        tmem_wait_ld();
        tc_fence_before();
        store_dq_row(dqkv, aq, pb, ph, prow, g, C, sh);
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
