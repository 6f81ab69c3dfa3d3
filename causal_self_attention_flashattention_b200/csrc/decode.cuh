// Decode attention: one new query row per (batch, head) against the keys and
// values already in the packed qkv buffer.
//
// The sampling loop of the GPT-2 reproduction generates one token at a time
// ("Let's reproduce GPT-2 (124M)" video description, chapter 00:37:02,
// generation loop); with the earlier rows' k and v kept, each step needs only
// the attention of the newest row t over rows 0..t. That is row t of the
// causal forward, so it is checked against the same definition.
//
// The work is one query row and up to T key rows per (b, h): 2*D*(t+1)
// multiply-adds against 4*D*(t+1) bytes of k and v, so it is bound by memory
// bandwidth and runs on the CUDA cores in fp32 (no tensor-core tile would be
// more than 1/128 full). Keys are split into 128-row chunks (split-K):
//   attn_decode_partial_kernel  one CTA (4 warps) per (chunk, h, b). One
//       thread issues two TMA box loads at once, the chunk's 128 k rows and
//       its 128 v rows (16 KiB each, the forward's packed-qkv tensor map,
//       128-byte swizzle, each on its own mbarrier), so every byte the CTA
//       needs is in flight from its first instruction and the scores start
//       as soon as the k rows land. At 36 KiB of shared memory per CTA (with
//       the alignment slack and the per-CTA reserve), six CTAs fit on an SM:
//       888 resident CTAs hold 28 MiB of loads in flight. Thread r scores key
//       r against q (held in registers) from shared memory; the block takes
//       its max and sum in base 2; and each warp accumulates p * v over its 32
//       keys, each lane owning two of the 64 columns. The four warps are
//       combined and the chunk's (max, sum, unnormalised o) goes to the
//       workspace.
//   attn_decode_combine_kernel  one CTA per (h, b): merges the chunks
//       (rescaling each by 2^(m_c - m)) into out (bf16) and the natural-log
//       lse; a programmatic dependent launch, so its CTAs are resident and
//       waiting when the partials land.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace decode {

constexpr int kChunk = 128;        // keys per CTA
constexpr int kWarps = 4;          // 32 keys per warp in the p * v step
constexpr int kPartialFloats = 2 + kD;  // m, l, o[D]

__host__ __device__ inline int num_chunks(int t) { return ceil_div(t + 1, kChunk); }

// Workspace: partials fp32 [B][H][chunks][2 + D] for chunks = ceil(T / 128).
__host__ __device__ inline size_t ws_bytes(int B, int T, int H) {
  return static_cast<size_t>(B) * H * num_chunks(T - 1) * kPartialFloats * sizeof(float);
}

struct alignas(1024) Smem {
  uint8_t k[kTileBytes];  // 128 rows x 128 bytes, 128-byte swizzle
  uint8_t v[kTileBytes];
  float p[kChunk];
  float red[2][kWarps];
  float o[kWarps][kD];
  uint64_t full_k, full_v;  // the chunk's k rows, v rows landed
  int abort;
};
constexpr size_t kSmemBytes = sizeof(Smem) + 1024;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Byte offset of 16-byte chunk c of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(kWarps * 32)
attn_decode_partial_kernel(const __grid_constant__ CUtensorMap map_qkv,
                           const __nv_bfloat16* __restrict__ qkv, int t,
                           float* __restrict__ partials, const AttnShape sh) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~uintptr_t(1023));
  // The combine kernel may be scheduled now; it waits for this grid's
  // writes before reading them.
  grid_dependents_launch();
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = sh.H * kD;
  const int c0 = chunk * kChunk;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full_k, 1);
    mbar_init(&sm.full_v, 1);
    sm.abort = 0;
    fence_barrier_init();
    mbar_arrive_expect_tx(&sm.full_k, kTileBytes);
    tma_load_3d(sm.k, &map_qkv, &sm.full_k, C + h * kD, c0, b);
    mbar_arrive_expect_tx(&sm.full_v, kTileBytes);
    tma_load_3d(sm.v, &map_qkv, &sm.full_v, 2 * C + h * kD, c0, b);
  }
  // q of row t (every thread reads the same 128 bytes), meanwhile.
  const size_t row_elems = static_cast<size_t>(3) * C;
  const uint4* qp = reinterpret_cast<const uint4*>(qkv + (static_cast<size_t>(b) * sh.T + t) * row_elems + h * kD);
  uint32_t q[32];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 w = __ldg(qp + c);
    q[4 * c] = w.x;
    q[4 * c + 1] = w.y;
    q[4 * c + 2] = w.z;
    q[4 * c + 3] = w.w;
  }
  __syncthreads();  // the barrier is initialised before anyone waits on it
  // The scores need only k; v is waited for before the p * v step.
  bool ok = mbar_wait(&sm.full_k, 0, kSiteDecode, &sm.abort);
  // Every thread leaves through the same barriers below; a thread whose wait
  // gave up computes on whatever is in shared memory and nothing is written.
  const int key = c0 + threadIdx.x;
  float s = -INFINITY;
  if (key <= t) {
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 w = *reinterpret_cast<const uint4*>(sm.k + sw128(threadIdx.x, c));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc0 = fmaf(__uint_as_float(q[4 * c + e] << 16), __uint_as_float(u[e] << 16), acc0);
        acc1 = fmaf(__uint_as_float(q[4 * c + e] & 0xFFFF0000u), __uint_as_float(u[e] & 0xFFFF0000u), acc1);
      }
    }
    s = (acc0 + acc1) * sh.scale_log2;
  }
  // Block max and sum in base 2.
  float m = warp_max(s);
  if (lane == 0) sm.red[0][warp] = m;
  __syncthreads();
  const float M = fmaxf(fmax3(sm.red[0][0], sm.red[0][1], sm.red[0][2]), sm.red[0][3]);
  const float p = key <= t ? exp2f(s - M) : 0.f;  // M is finite: key c0 <= t always
  sm.p[threadIdx.x] = p;
  const float l = warp_sum(p);
  if (lane == 0) sm.red[1][warp] = l;
  __syncthreads();
  ok = mbar_wait(&sm.full_v, 0, kSiteDecode, &sm.abort) && ok;
  // o[2*lane .. 2*lane+1] = sum over this warp's 32 keys of p * v.
  float o0 = 0.f, o1 = 0.f;
  const int cpair = lane >> 2;         // 16-byte chunk holding columns 2*lane, 2*lane+1
  const int wofs = (lane & 3) * 4;     // byte offset of the pair within the chunk
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const int r = warp * 32 + i;
    const float pr = sm.p[r];
    const uint32_t vv = *reinterpret_cast<const uint32_t*>(sm.v + sw128(r, cpair) + wofs);
    o0 = fmaf(pr, __uint_as_float(vv << 16), o0);
    o1 = fmaf(pr, __uint_as_float(vv & 0xFFFF0000u), o1);
  }
  sm.o[warp][2 * lane] = o0;
  sm.o[warp][2 * lane + 1] = o1;
  __syncthreads();
  if (__syncthreads_or(!ok)) {
    // A wait gave up: nothing is written; the loads still in flight are
    // waited for (bounded) before the CTA's shared memory goes away.
    if (threadIdx.x == 0) {
      drain_wait(&sm.full_k, 0, kSiteDecode);
      drain_wait(&sm.full_v, 0, kSiteDecode);
    }
  } else {
    float* out = partials + ((static_cast<size_t>(b) * sh.H + h) * gridDim.x + chunk) * kPartialFloats;
    if (threadIdx.x < kD)
      out[2 + threadIdx.x] = (sm.o[0][threadIdx.x] + sm.o[1][threadIdx.x]) +
                             (sm.o[2][threadIdx.x] + sm.o[3][threadIdx.x]);
    if (threadIdx.x == 0) {
      out[0] = M;
      out[1] = (sm.red[1][0] + sm.red[1][1]) + (sm.red[1][2] + sm.red[1][3]);
    }
  }
}

// One CTA of 64 threads (one per column) per (h, b). The chunks are read in
// batches of 8 with independent loads (one round trip to L2 per batch, not
// one per chunk) and merged against a running max: a batch raises the max
// M to include its chunks, rescales the sums so far by 2^(M_old - M), and
// adds its chunks (each rescaled by 2^(m_c - M)) in chunk order. Rows of at
// most 8 chunks are one batch. Launched as a programmatic dependent of the
// partial kernel: the CTAs may start while the partials are still being
// written, and wait for them (griddepcontrol.wait) before the first read.
__global__ void __launch_bounds__(kD)
attn_decode_combine_kernel(const float* __restrict__ partials, int n_chunks,
                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                           const AttnShape sh) {
  grid_dependency_wait();
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float* p = partials + (static_cast<size_t>(b) * sh.H + h) * n_chunks * kPartialFloats;
  constexpr int kBatch = 8;
  float M = -INFINITY, L = 0.f, o = 0.f;
  for (int c0 = 0; c0 < n_chunks; c0 += kBatch) {
    float mc[kBatch], lc[kBatch], oc[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const bool in = c0 + i < n_chunks;
      const float* pc = p + (c0 + i) * kPartialFloats;
      mc[i] = in ? pc[0] : -INFINITY;
      lc[i] = in ? pc[1] : 0.f;
      oc[i] = in ? pc[2 + d] : 0.f;
    }
    float Mb = M;
#pragma unroll
    for (int i = 0; i < kBatch; ++i) Mb = fmaxf(Mb, mc[i]);
    if (M != -INFINITY) {
      const float w = exp2f(M - Mb);
      L *= w;
      o *= w;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (mc[i] == -INFINITY) continue;
      const float w = exp2f(mc[i] - Mb);
      L = fmaf(lc[i], w, L);
      o = fmaf(oc[i], w, o);
    }
    M = Mb;
  }
  out[(static_cast<size_t>(b) * sh.H + h) * kD + d] = __float2bfloat16_rn(o / L);
  if (d == 0) lse[static_cast<size_t>(b) * sh.H + h] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace decode
}  // namespace ga
