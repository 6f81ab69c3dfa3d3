// Shapes, tiling constants and the packed-QKV addressing shared by the
// attention kernels.
//
// Packed QKV: element (b, t, s, h, d) of qkv (B, T, 3, H, D) sits at
//     (((b*T + t)*3 + s)*H + h)*D + d,   s = 0 (q), 1 (k), 2 (v).
// The TMA maps view it as a 3-D tensor {3*H*D, T, B} (innermost first), so the
// 128-row tile of slot s, head h, rows [t0, t0+128) of batch b is the box at
// coordinates {s*H*D + h*D, t0, b}. Rows past T read as zero.
// out, dout (B, T, H, D) are viewed as {H*D, T, B} the same way.
#pragma once

#include <cstdint>

namespace ga {

constexpr int kD = 64;         // head dimension (GPT-2: 768 / 12)
constexpr int kBlockM = 128;   // query rows per tile
constexpr int kBlockN = 128;   // key rows per tile
constexpr int kTileBytes = kBlockM * kD * 2;  // one 128 x 64 bf16 tile = 16 KiB

// Wait-site codes reported in the device status word (high 32 bits).
enum WaitSite : uint32_t {
  kSiteFwdProducer = 0x101,
  kSiteFwdMma = 0x102,
  kSiteFwdSoftmax = 0x103,
  kSiteFwdConvert = 0x104,
  kFwdValueRange = 0x1F0,  // a V entry outside the fp16 range (|v| > 65504, inf, NaN)
  kSiteDqProducer = 0x201,
  kSiteDqMma = 0x202,
  kSiteDqSoftmax = 0x203,
  kSiteDkvProducer = 0x301,
  kSiteDkvMma = 0x302,
  kSiteDkvSoftmax = 0x303,
  kSiteFusedProducer = 0x401,
  kSiteFusedMma = 0x402,
  kSiteFusedSoftmax = 0x403,
  kSiteFusedDq = 0x404,  // waiting for earlier key tiles' dQ sums
  kSiteDecode = 0x701,  // the decode kernel's wait for its k and v chunk
  kSiteLinearProducer = 0x601,
  kSiteLinearMma = 0x602,
  kSiteLinearEpilogue = 0x603,
  kSiteSelftestWait = 0x501,  // the self-test's wait that nothing completes
  kSiteSelftestPeer = 0x502,  // the self-test's second waiter (winds down on the abort flag)
};

struct AttnShape {
  int B, T, H;
  float scale_log2;   // scale * log2(e): logits in base-2 units
  float scale;        // softmax scale (1/sqrt(D) for GPT-2)
};

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Work item of a persistent CTA in round r: boustrophedon order over the
// grid, r*G + c on even rounds and r*G + (G - 1 - c) on odd ones. With items
// sorted heaviest first this evens out the CTAs' totals (for the GPT-2 shapes
// the busiest CTA gets 1.01-1.07x the mean instead of up to 1.16x for plain
// striding). The result may be >= the item count on the last round.
__device__ __forceinline__ int snake_item(int r, int grid, int cta) {
  return r * grid + ((r & 1) ? (grid - 1 - cta) : cta);
}

// A deal of work items to the CTAs of one launch, computed on the host and
// passed by value (a kernel parameter): CTA c runs items base + item[t] for t
// in [start[c], start[c + 1]), in that order, at most kSchedSlots of them.
// Every launch copies the whole parameter, so kernels come with a small and a
// large table, and the host picks the smaller one that holds the deal.
constexpr int kSchedMaxCtas = 160;
constexpr int kSchedSlots = 64;
template <int kItems>
struct ItemSchedule {
  int base;
  uint16_t start[kSchedMaxCtas + 1];
  uint16_t item[kItems];
};

// Copies this CTA's items into items[0 .. n) and n into items[kSchedSlots];
// every thread of the block takes part, and a barrier must follow before the
// list is read.
template <int kItems>
__device__ __forceinline__ void load_item_list(const ItemSchedule<kItems>& sched, int* items) {
  const int t0 = sched.start[blockIdx.x];
  const int n = min(sched.start[blockIdx.x + 1] - t0, kSchedSlots);
  if (threadIdx.x == 0) items[kSchedSlots] = n;
  for (int t = threadIdx.x; t < n; t += blockDim.x) items[t] = sched.base + sched.item[t0 + t];
}

}  // namespace ga
