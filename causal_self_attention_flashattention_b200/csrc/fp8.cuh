// Per-tensor e4m3 quantisation of the packed q, k, v for the FP8 forward.
//
// The llm.c page plans FP8 training ("Réimplémenter à bas coût le modèle
// GPT-2 avec llm.c", FAQ entry on FP8). Each of the three slots of qkv
// (B, T, 3, H, D) gets one scale, chosen so that its largest magnitude maps to
// 448, the largest e4m3 value:
//     amax_s = max |x|,  scale_s = 448 / amax_s,  x8 = e4m3_rn(x * scale_s),
//     dequant_s = amax_s / 448   (1 and 1 when amax_s = 0),
// every step one correctly rounded fp32 operation. Three launches:
//   fp8_zero_kernel     clears the amax words;
//   fp8_amax_kernel     grid-stride max |x| per slot (atomicMax on the bits of
//                       non-negative floats, which order like the floats);
//   fp8_quantize_kernel scales, rounds (cvt.rn.satfinite: to nearest even,
//                       finite) and writes the bytes; block 0 writes dequant.
// Both passes read qkv in 16-byte pieces (8 bf16 of one slot: C = 64 H is a
// multiple of 8).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace fp8 {

constexpr float kE4m3Max = 448.f;
constexpr int kThreads = 256;

// Layout of the caller's fp32[8] scale buffer.
constexpr int kDequantOffset = 0;  // [0..2] dequantisation multipliers (output)
constexpr int kAmaxOffset = 4;     // [4..6] amax bits (scratch)

__global__ void fp8_zero_kernel(float* __restrict__ scales) {
  if (threadIdx.x < 3) reinterpret_cast<uint32_t*>(scales)[kAmaxOffset + threadIdx.x] = 0u;
}

__global__ void __launch_bounds__(kThreads)
fp8_amax_kernel(const uint4* __restrict__ qkv, long long n_chunks, int C, float* __restrict__ scales) {
  float mx[3] = {0.f, 0.f, 0.f};
  const int row_chunks = 3 * C / 8;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int slot = static_cast<int>(i % row_chunks) / (C / 8);
    const uint4 v = qkv[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      m = fmax3(m, fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
    mx[0] = slot == 0 ? fmaxf(mx[0], m) : mx[0];
    mx[1] = slot == 1 ? fmaxf(mx[1], m) : mx[1];
    mx[2] = slot == 2 ? fmaxf(mx[2], m) : mx[2];
  }
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    float m = mx[s];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0 && m > 0.f)
      atomicMax(reinterpret_cast<unsigned int*>(scales) + kAmaxOffset + s, __float_as_uint(m));
  }
}

__device__ __forceinline__ float slot_scale(const float* scales, int s) {
  const float amax = scales[kAmaxOffset + s];
  return amax > 0.f ? kE4m3Max / amax : 1.f;
}

__global__ void __launch_bounds__(kThreads)
fp8_quantize_kernel(const uint4* __restrict__ qkv, uint2* __restrict__ qkv8, long long n_chunks,
                    int C, float* __restrict__ scales) {
  const float sc[3] = {slot_scale(scales, 0), slot_scale(scales, 1), slot_scale(scales, 2)};
  if (blockIdx.x == 0 && threadIdx.x < 3) {
    const float amax = scales[kAmaxOffset + threadIdx.x];
    scales[kDequantOffset + threadIdx.x] = amax > 0.f ? amax / kE4m3Max : 1.f;
  }
  const int row_chunks = 3 * C / 8;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int slot = static_cast<int>(i % row_chunks) / (C / 8);
    const float f = slot == 0 ? sc[0] : (slot == 1 ? sc[1] : sc[2]);
    const uint4 v = qkv[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_e4m3(__uint_as_float(w[e] << 16) * f, __uint_as_float(w[e] & 0xFFFF0000u) * f);
    qkv8[i] = make_uint2(o[0] | (o[1] << 16), o[2] | (o[3] << 16));
  }
}

}  // namespace fp8
}  // namespace ga
