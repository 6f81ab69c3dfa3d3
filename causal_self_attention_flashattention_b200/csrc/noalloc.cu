// gpt2_attn_bwd_noalloc: the backward with its scratch buffer in static device
// memory, for callers that cannot allocate device memory.
//
// gpt2_attn_bwd needs a caller-provided workspace (Delta, fp32 (B,H,T)). Some
// callers have no way to provide one: a plugin handed only its input and output
// tensors by a host application that owns all device memory, or a program that
// reserves the GPU's memory once at start-up and may not call cudaMalloc (or pay
// for its implicit synchronisation) afterwards. This entry point keeps Delta in
// a fixed array that lives in the library's own device image instead.
//
// The array is loaded with the library on every GPU that runs it and stays
// resident until the process exits: kMaxDeltaElems floats (4 MiB) per device.
// It is shared by every call. The dQ step rewrites every Delta value a call
// reads before the call reads it, so nothing has to be cleared between
// calls, but two calls whose work overlaps on the GPU (different streams, or
// different host threads on one device) race on the array.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gpt2attn.h"
#include "checks.h"

namespace {

constexpr size_t kMaxDeltaElems = size_t(1) << 20;  // B*H*T <= 1,048,576

// Device-side scratch for Delta. In host code this name is only a host-side
// stand-in for the symbol, never a device address: the kernels receive the
// address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) float g_noalloc_delta[kMaxDeltaElems];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_delta_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the array.
float* delta_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_delta_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_delta) != cudaSuccess || p == nullptr) return nullptr;
    g_delta_ptr[dev] = static_cast<float*>(p);
  }
  return g_delta_ptr[dev];
}

}  // namespace

// Every argument is checked here, with the same rules as every other entry
// point (checks.h), before the first of the two launches; only the size limit
// of the static array is this entry point's own.
extern "C" ga_status gpt2_attn_bwd_noalloc(const void* qkv, const void* out, const void* dout,
                                           const float* lse, void* dqkv, int B, int T, int H,
                                           int D, float scale, gpt2attn_stream_t stream) {
  ga_status st = ga_host::check_shape(B, T, H, D);
  if (st != GA_OK) return st;
  if (static_cast<long double>(B) * H * T > static_cast<long double>(kMaxDeltaElems))
    return GA_ERR_WORKSPACE;
  if (qkv == nullptr || out == nullptr || dout == nullptr || lse == nullptr || dqkv == nullptr)
    return GA_ERR_INVALID_ARG;
  if ((st = ga_host::check_scale(scale)) != GA_OK) return st;
  if (!ga_host::aligned16(qkv) || !ga_host::aligned16(out) || !ga_host::aligned16(dout) ||
      !ga_host::aligned16(lse) || !ga_host::aligned16(dqkv))
    return GA_ERR_ALIGNMENT;
  float* delta = delta_scratch();
  if (delta == nullptr) return GA_ERR_CUDA;
  if ((st = gpt2_attn_bwd_dq(qkv, out, dout, lse, delta, dqkv, B, T, H, D, scale, stream)) !=
      GA_OK)
    return st;
  return gpt2_attn_bwd_dkdv(qkv, dout, lse, delta, dqkv, B, T, H, D, scale, stream);
}
