// Argument checks shared by the library's entry points (defined in
// gpt2attn.cu). Every entry point validates its arguments with these before
// any CUDA call, so that all of them accept and refuse the same shapes,
// scales and pointers.
#pragma once

#include "gpt2attn.h"

namespace ga_host {

// B, T, H >= 1 and D >= 1 (GA_ERR_INVALID_ARG otherwise), D == 64
// (GA_ERR_UNSUPPORTED otherwise), and B*T*3*H*D below 2^31 elements.
ga_status check_shape(int B, int T, int H, int D);

// scale finite and > 0 (GA_ERR_INVALID_ARG otherwise).
ga_status check_scale(float scale);

// The pointer is 16-byte aligned (every TMA base and vector access needs it).
bool aligned16(const void* p);

}  // namespace ga_host
