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
// more than 1/128 full). Keys are split into 256-row chunks (split-K):
//   attn_decode_partial_kernel  one CTA (4 warps) per (chunk, h, b). The
//       chunk's v rows are copied to shared memory (cp.async, 16 bytes per
//       copy) while each warp scores its 64 keys, so both loads are in flight
//       at once. Eight lanes read one 128-byte k row together (each 16 bytes
//       against its eighth of q, then three shuffles), so a warp's load
//       instruction covers four whole rows. Each warp takes its max and sum in
//       base 2 and accumulates p * v from shared memory, each lane owning two
//       of the 64 columns; the four warps are then combined, and the chunk's
//       (max, sum, unnormalised o) goes to the workspace.
//   attn_decode_combine_kernel  one CTA per (h, b): merges the chunks
//       (rescaling each by 2^(m_c - m)) into out (bf16) and the natural-log lse.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace decode {

constexpr int kChunk = 256;        // keys per CTA
constexpr int kWarps = 4;          // 64 keys per warp
constexpr int kPartialFloats = 2 + kD;  // m, l, o[D]

__host__ __device__ inline int num_chunks(int t) { return ceil_div(t + 1, kChunk); }

// Workspace: partials fp32 [B][H][chunks][2 + D] for chunks = ceil(T / 256).
__host__ __device__ inline size_t ws_bytes(int B, int T, int H) {
  return static_cast<size_t>(B) * H * num_chunks(T - 1) * kPartialFloats * sizeof(float);
}

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

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}

__global__ void __launch_bounds__(kWarps * 32)
attn_decode_partial_kernel(const __nv_bfloat16* __restrict__ qkv, int t,
                           float* __restrict__ partials, const AttnShape sh) {
  __shared__ float m_s[kWarps], l_s[kWarps];
  __shared__ float s_s[kWarps][64];  // the warps' scores
  __shared__ float o_s[kWarps][kD];
  __shared__ __align__(16) __nv_bfloat16 v_s[kChunk][kD];  // 32 KiB
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_elems = static_cast<size_t>(3) * sh.H * kD;  // one (b, t) row of qkv
  const __nv_bfloat16* base = qkv + static_cast<size_t>(b) * sh.T * row_elems + h * kD;
  // The chunk's v rows (those <= t), 8 sixteen-byte pieces per row.
  {
    const int c0 = chunk * kChunk;
    const int rows = min(kChunk, t + 1 - c0);
    const __nv_bfloat16* vsrc = base + 2 * sh.H * kD + static_cast<size_t>(c0) * row_elems;
    for (int idx = threadIdx.x; idx < rows * (kD / 8); idx += kWarps * 32) {
      const int rr = idx >> 3, piece = idx & 7;
      cp_async16(&v_s[rr][8 * piece], vsrc + rr * row_elems + 8 * piece);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // This lane's eighth of q: columns [8 * piece, 8 * piece + 8).
  const int piece = lane & 7;
  const uint4 qw = __ldg(reinterpret_cast<const uint4*>(base + t * row_elems) + piece);
  const uint32_t q[4] = {qw.x, qw.y, qw.z, qw.w};

  // Scores of this warp's 64 keys, four rows per step: lanes 8r..8r+7 read
  // row r of the step, 16 bytes each.
  const int k0 = chunk * kChunk + warp * 64;
  const __nv_bfloat16* kbase = base + sh.H * kD;  // the k slot
#pragma unroll 4
  for (int g = 0; g < 16; ++g) {
    const int key = k0 + 4 * g + (lane >> 3);
    float part = 0.f;
    if (key <= t) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(kbase + key * row_elems) + piece);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        part = fmaf(__uint_as_float(q[e] << 16), __uint_as_float(u[e] << 16), part);
        part = fmaf(__uint_as_float(q[e] & 0xFFFF0000u), __uint_as_float(u[e] & 0xFFFF0000u), part);
      }
    }
    part += __shfl_xor_sync(0xffffffffu, part, 4);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    if (piece == 0) s_s[warp][4 * g + (lane >> 3)] = key <= t ? part * sh.scale_log2 : -INFINITY;
  }
  __syncwarp();
  const float sa = s_s[warp][lane], sb = s_s[warp][32 + lane];
  const float m = warp_max(fmaxf(sa, sb));
  // A warp whose keys all lie past t contributes nothing (m = -inf).
  const float pa = m == -INFINITY ? 0.f : exp2f(sa - m);
  const float pb = m == -INFINITY ? 0.f : exp2f(sb - m);
  const float l = warp_sum(pa + pb);

  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();  // every thread's v copies have landed

  // o[2*lane .. 2*lane+1] = sum over the warp's keys of p * v.
  float o0 = 0.f, o1 = 0.f;
  const int n_keys = min(64, t + 1 - k0);  // <= 0 when the warp has no keys
  const int r0 = warp * 64;                 // the warp's first row within v_s
#pragma unroll 8
  for (int i = 0; i < n_keys; ++i) {
    const float p = __shfl_sync(0xffffffffu, i < 32 ? pa : pb, i & 31);
    const float2 vf =
        __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v_s[r0 + i][2 * lane]));
    o0 = fmaf(p, vf.x, o0);
    o1 = fmaf(p, vf.y, o1);
  }
  if (lane == 0) {
    m_s[warp] = m;
    l_s[warp] = l;
  }
  o_s[warp][2 * lane] = o0;
  o_s[warp][2 * lane + 1] = o1;
  __syncthreads();

  // Combine the four warps: rescale each by 2^(m_w - M).
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, m_s[w]);
  float* out = partials + ((static_cast<size_t>(b) * sh.H + h) * gridDim.x + chunk) * kPartialFloats;
  if (threadIdx.x < kD) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (m_s[w] != -INFINITY) o = fmaf(o_s[w][threadIdx.x], exp2f(m_s[w] - M), o);
    out[2 + threadIdx.x] = o;
  }
  if (threadIdx.x == 0) {
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (m_s[w] != -INFINITY) L = fmaf(l_s[w], exp2f(m_s[w] - M), L);
    out[0] = M;
    out[1] = L;
  }
}

// One CTA of 64 threads (one per column) per (h, b).
__global__ void __launch_bounds__(kD)
attn_decode_combine_kernel(const float* __restrict__ partials, int n_chunks,
                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                           const AttnShape sh) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  const float* p = partials + (static_cast<size_t>(b) * sh.H + h) * n_chunks * kPartialFloats;
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, p[c * kPartialFloats]);
  float L = 0.f, o = 0.f;
  for (int c = 0; c < n_chunks; ++c) {
    const float mc = p[c * kPartialFloats];
    if (mc == -INFINITY) continue;
    const float w = exp2f(mc - M);
    L = fmaf(p[c * kPartialFloats + 1], w, L);
    o = fmaf(p[c * kPartialFloats + 2 + d], w, o);
  }
  out[(static_cast<size_t>(b) * sh.H + h) * kD + d] = __float2bfloat16_rn(o / L);
  if (d == 0) lse[static_cast<size_t>(b) * sh.H + h] = (M + log2f(L)) * 0.69314718055994531f;
}

}  // namespace decode
}  // namespace ga
