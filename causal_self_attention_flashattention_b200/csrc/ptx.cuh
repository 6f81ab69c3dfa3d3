// Thin inline-PTX wrappers for the sm_100a features the attention kernels use:
// mbarriers (with bounded waits), TMA tensor loads, tcgen05 tensor-memory
// allocation, MMA, commit, load/store and fences, plus a few ALU helpers.
//
// Every wait in this library is bounded: after kWaitTimeoutNs of polling the
// waiting thread records the site in the device status word, raises the
// CTA's abort flag and returns false. The caller then winds its role down.
// No wait in these kernels can spin forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace ga {

// ---------------------------------------------------------------------------
// Status word shared by all kernels of the library.
// ---------------------------------------------------------------------------
static __device__ unsigned long long g_device_status;

constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Records the first failure: high 32 bits = site code, low = block index.
__device__ __forceinline__ void record_failure(uint32_t site) {
  unsigned long long v = (static_cast<unsigned long long>(site) << 32) | blockIdx.x;
  atomicCAS(&g_device_status, 0ull, v);
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may sleep up to `ns` nanoseconds for the
// phase to complete instead of returning at once; a sleeping thread takes no
// issue slots from the warps that do the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

constexpr uint32_t kWaitSleepNs = 20000;  // per try; the timeout is checked every 8 tries

// Non-blocking check: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most
// `limit_ns`. Returns false (after recording `site` and raising `*abort`) when
// the limit passes, or (without recording) when another role of the CTA has
// already raised `*abort`.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, uint32_t site,
                                                volatile int* abort, uint64_t limit_ns) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(addr, parity, kWaitSleepNs)) return true;
    if ((it & 7u) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > limit_ns) {
        record_failure(site);
        *abort = 1;
        return false;
      }
    }
  }
}

// The wait every kernel of the library uses: mbar_wait_limit with the 2 s
// limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t site,
                                          volatile int* abort) {
  return mbar_wait_limit(bar, parity, site, abort, kWaitTimeoutNs);
}

// Wait used while winding down: ignores the abort flag, still bounded.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint32_t site) {
  volatile int no_abort = 0;
  return mbar_wait(bar, parity, site, &no_abort);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch
// ---------------------------------------------------------------------------
// Lets the grid launched after this one on the stream (with the programmatic
// stream serialization attribute) be scheduled before this grid finishes.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the grids this one depends on have completed and their memory
// writes are visible. Returns at once for a grid launched without the
// attribute.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs: a two-CTA cluster whose tensor-core products span both SMs
// (tcgen05 .cta_group::2). The even CTA (rank 0) issues the products; each
// CTA holds its half of the operands and of the accumulator.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of both CTAs arrives and waits (all CTAs of a cluster are
// resident together, so it completes once every thread reaches it).
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The shared::cluster address of `local`'s counterpart in the CTA of cluster
// rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}

// Arrive (release, cluster scope) on an mbarrier given by its shared::cluster
// address, possibly in the other CTA.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr)
               : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// 2-D tiled load into this CTA's shared memory whose completion is counted on
// the mbarrier at `bar_cluster_addr` (the even CTA's, for either CTA of the
// pair). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}

// D (+)= A B over the pair: the descriptors address this CTA's halves; the
// partner's halves sit at the same shared-memory offsets, and each CTA's
// tensor memory holds its 128 rows of D. Issued by one thread of the even CTA.
__device__ __forceinline__ void mma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on the mbarrier at the same offset in both CTAs of the pair once
// the pair's products issued so far have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  const uint16_t both = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(both)
      : "memory");
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load of one box into shared memory; completion is signalled on
// `bar` as transaction bytes. Coordinates are element indices, innermost first.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 2-D tiled load of one box into shared memory (same completion mechanism).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 3-D tiled store of one box from shared memory to global memory (bulk
// group completion). Boxes that reach past the tensor's edge are clipped.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 2-D tiled store of one box from shared memory (bulk group completion);
// boxes reaching past the tensor's edge are clipped.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until every committed bulk store has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until all but the most recent committed bulk store have finished
// reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Waits until every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor-core MMA
// ---------------------------------------------------------------------------
// Allocation is warp-wide; the TMEM base address is written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T-style product described by the descriptors.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same with the A operand read from tensor memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem] with 8-bit (e4m3) operands: 32 elements of K
// per instruction.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

#define GA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                 "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define GA_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                 "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 lanes x 32 bits, 32 consecutive columns: thread t of the warp gets
// columns [col, col+32) of lane (warp's lane quarter base + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : GA_R8(0), GA_R8(8), GA_R8(16), GA_R8(24)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : GA_R8(0), GA_R8(8)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      GA_W8(0)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      GA_W8(0), GA_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      GA_W8(0), GA_W8(8), GA_W8(16), GA_W8(24)
      : "memory");
}

#undef GA_R8
#undef GA_W8

// ---------------------------------------------------------------------------
// Descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor for a 128-byte-swizzled tile whose 8-row
// swizzle atoms are 1024 bytes apart (the layout TMA writes for a box whose
// inner extent is 128 bytes). Fields: start address >> 4 in bits [0,14),
// leading byte offset >> 4 in [16,30), stride byte offset >> 4 in [32,46),
// descriptor version 1 in [46,48), swizzle mode 2 (128B) in [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// Shared-memory descriptor for a K-major tile without swizzle: 8-row x 16-byte
// core matrices stored contiguously (row i at +16i), `lbo_bytes` apart along
// K and `sbo_bytes` apart along M/N. Same fields as above, swizzle mode 0.
__device__ __forceinline__ uint64_t smem_desc_noswizzle(uint32_t saddr, uint32_t lbo_bytes,
                                                        uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  return d;
}

// Shared-memory descriptor for a K-major tile with 64-byte rows and the
// 64-byte swizzle (8-row atoms 512 bytes apart), as TMA writes a box whose
// inner extent is 64 bytes: swizzle mode 4 in [61,64), otherwise as above.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 4ull << 61;
  return d;
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B (format code 0)
// and fp32 accumulate, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with bf16 inputs and fp32 accumulate.
// a_mn / b_mn select MN-major (1) or K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                                  // D format: f32
         | (1u << 7)                                // A format: bf16
         | (1u << 10)                               // B format: bf16
         | (static_cast<uint32_t>(a_mn) << 15)      // A major
         | (static_cast<uint32_t>(b_mn) << 16)      // B major
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// Same with fp16 A and B (format code 0), fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// ALU helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Packs two floats to bf16x2 (round to nearest even); `lo` goes to the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Packs two floats to f16x2 (round to nearest even); `lo` goes to the low half.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------------------
// Float -> half conversions on the FMA/ALU pipes
// ---------------------------------------------------------------------------
// cvt.rn.{f16,bf16}x2.f32 runs on the same pipe as ex2.approx, which the
// softmax keeps saturated. These equivalents use the FMA and integer pipes.

// (a0 * s, a1 * s) in one packed fp32 multiply; round to nearest, subnormals
// kept.
__device__ __forceinline__ void mul2(float a0, float a1, float s, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, r;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %4};\n\t"
      "mul.rn.f32x2 r, a, b;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(s));
}

// (a0 * b + c, a1 * b + c) in one packed fp32 fused multiply-add.
__device__ __forceinline__ void fma2(float a0, float a1, float b, float c, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, c, r;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %4};\n\t"
      "mov.b64 c, {%5, %5};\n\t"
      "fma.rn.f32x2 r, a, b, c;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (a0 * b0 + c0, a1 * b1 + c1) in one packed fp32 fused multiply-add.
__device__ __forceinline__ void fma2v(float a0, float a1, float b0, float b1, float c0, float c1,
                                      float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, c, r;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 r, a, b, c;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (a0 * b0, a1 * b1) in one packed fp32 multiply.
__device__ __forceinline__ void mul2v(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  asm("{\n\t.reg .b64 a, b, r;\n\t"
      "mov.b64 a, {%2, %3};\n\t"
      "mov.b64 b, {%4, %5};\n\t"
      "mul.rn.f32x2 r, a, b;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// (a0 + b0, a1 + b1) in one packed fp32 add.
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 a, a, b;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

// 2^y for a pair of floats on the FMA/ALU pipes instead of the 16/clk exp
// unit. y = n + f with n = rint(y) (adding 1.5 * 2^23 rounds y to an integer
// that lands in the low mantissa bits), 2^f from a cubic, and n added to the
// exponent field. The cubic was fitted to 2^f on [-1/2, 1/2] by least squares
// on Chebyshev nodes, reweighted toward equal ripple (Lawson's iteration); its
// largest relative error there is 7.5e-5. y is clamped to >= -125 first, so
// the exponent never wraps: -inf and very negative y give a value below
// 2^-125 instead of 0.
constexpr float kExp2Poly0 = 0.9999280571937561f;
constexpr float kExp2Poly1 = 0.6932609677314758f;
constexpr float kExp2Poly2 = 0.2426111251115799f;
constexpr float kExp2Poly3 = 0.0551716648042202f;

__device__ __forceinline__ void exp2_poly2(float y0, float y1, float& p0, float& p1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  const float a0 = fmaxf(y0, -125.f), a1 = fmaxf(y1, -125.f);
  float t0 = a0, t1 = a1;
  add2(t0, t1, kRound, kRound);
  float n0 = t0, n1 = t1;
  add2(n0, n1, -kRound, -kRound);
  float f0, f1;
  fma2v(n0, n1, -1.f, -1.f, a0, a1, f0, f1);  // f = a - n, in [-1/2, 1/2]
  float q0, q1;
  fma2(f0, f1, kExp2Poly3, kExp2Poly2, q0, q1);
  fma2v(q0, q1, f0, f1, kExp2Poly1, kExp2Poly1, q0, q1);
  fma2v(q0, q1, f0, f1, kExp2Poly0, kExp2Poly0, q0, q1);
  // bits(t) << 23 == n << 23 (mod 2^32): the rounding constant's own bits
  // shift out.
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// fp16 bits of a float x in [0, 65504]: x * 2^-112 moves the exponent bias
// from 127 to 15, so bits [13, 29) of the product are the fp16 encoding,
// subnormals included. The factor is 2^-112 (1 + 3 * 2^-13) rather than
// 2^-112: for a significand f in [1, 2) it adds 3f/8 of an fp16 unit in the
// last place before the 13 low bits are dropped, so truncating rounds to one
// of the two fp16 values around x (up when the dropped part exceeds
// 1 - 3f/8 of a unit) with an error below 3/4 of a unit and a mean of about
// +0.04 of a unit over log-uniform x, without the two integer adds a half-up
// rounding takes.
constexpr float kF32ToF16Scale = 1.9266352409977292e-34f;  // 2^-112 (1 + 3 * 2^-13)

__device__ __forceinline__ uint32_t pack_f16_nonneg(float lo, float hi) {
  float m0, m1;
  mul2(lo, hi, kF32ToF16Scale, m0, m1);
  const uint32_t b0 = __float_as_uint(m0);
  const uint32_t b1 = __float_as_uint(m1);
  return (b0 >> 13) | ((b1 << 3) & 0xFFFF0000u);
}

// Per fp16 half: the larger magnitude of a and b (its sign is the xor of the
// signs, which callers ignore); a NaN in either input gives NaN.
__device__ __forceinline__ uint32_t max_abs_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Magnitude bits of an fp16 at or above this: inf or NaN.
constexpr uint32_t kF16InfBits = 0x7C00u;

// Per 16-bit half: the larger of a and b as unsigned integers.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// bf16 magnitude bits (per half) at or above this: |v| > 65280, the largest
// bf16 that fp16 holds (the next bf16, 65536, is beyond fp16's 65504), or inf,
// or NaN.
constexpr uint32_t kBf16BeyondF16 = 0x4780u;

// A pair of bf16 values (low half first) to a pair of fp16 values with
// integer operations only, leaving the exp unit to the softmax. A bf16 with
// biased exponent e and mantissa m is 2^(e-127) (1 + m/128); its fp16 has
// exponent e - 112 and mantissa m << 3, i.e. fp16 magnitude bits =
// (bf16 magnitude bits - (112 << 7)) << 3. Both halves go through one 32-bit
// multiply-add: (mag - 0x38003800) * 8 == mag * 8 + 0x3FFE4000 (mod 2^32),
// with no carry or borrow between the halves while each half's magnitude lies
// in [0x3800, 0x477F]; magnitudes below are clamped up to 0x3800, and above
// it the range tracker is raised (the pair's value is then unspecified).
// Results:
//   2^-14 <= |v| <= 65280   exact (every such bf16 is an fp16 normal);
//   |v| < 2^-15             +-0 (the clamp maps it to 0x3800, i.e. fp16 0);
//   2^-15 <= |v| < 2^-14    an fp16 subnormal within 2^-15 of v;
//   |v| > 65280, inf, NaN   unspecified, and `rng` (a running per-half max of
//                           the magnitude bits) reaches kBf16BeyondF16.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t u, uint32_t& rng) {
  const uint32_t mag = u & 0x7FFF7FFFu;
  rng = max_u16x2(rng, mag);
  const uint32_t clamped = max_u16x2(mag, 0x38003800u);
  return (clamped * 8u + 0x3FFE4000u) | (u & 0x80008000u);
}

// Two e4m3 values (bytes 0 and 1, or 2 and 3, of `w`, picked by `sel`) as an
// fp16 pair equal to the e4m3 values times 2^-8, with integer operations
// only. An e4m3 byte s.eeee.mmm (exponent bias 7) becomes the fp16 bits
// s.0eeee.mmm0000000 (exponent bias 15): the exponent field keeps its value,
// so every value, subnormals included, is scaled by exactly 2^(7-15). The
// sign moves from bit 7 to bit 8 of the 16-bit lane by adding the byte's own
// top bit to it (no carry leaves the lane), then the lane shifts by 7.
// `sel` is 0x4140 for bytes 0, 1 and 0x4342 for bytes 2, 3.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_scaled(uint32_t w, uint32_t sel) {
  uint32_t t;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(t) : "r"(w), "r"(sel));
  return (t + (t & 0x00800080u)) << 7;
}

// Two floats to an e4m3 pair (round to nearest even, saturating to +-448);
// `lo` goes to the low byte.
__device__ __forceinline__ uint16_t pack_e4m3(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Warpgroup-wide register budget changes (all four warps of a warpgroup
// execute the same one). The budgets of all warpgroups must add up to no more
// than the block's launch allocation, or setmaxnreg.inc would wait forever.
template <uint32_t kRegs>
__device__ __forceinline__ void regs_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <uint32_t kRegs>
__device__ __forceinline__ void regs_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// Named barrier among `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace ga
