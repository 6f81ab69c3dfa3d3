// Forward kernel: out = softmax(scale * Q K^T + causal mask) V and the row
// logsumexp, with the T x T matrix never leaving tensor memory / registers.
//
// Flash attention "never stores the full attention matrix" ("Let's reproduce
// GPT-2 (124M)" video summary page, glossary table, row "flash attention").
// This kernel does that as follows on sm_100a:
//
//   * Work item = one (batch, head) and a pair of adjacent 128-row query tiles
//     (rows [256p, 256p+256)). Items run heaviest first over a persistent grid.
//   * Warp 8 (TMA): loads the two Q tiles once per item (double-buffered
//     across items) and streams the 128-row K and V tiles j = 0..2p+1 through a
//     4-stage shared-memory ring.
//   * Warps 9 and 10 (MMA, one thread each, one per warpgroup q): S_q = Q K_j^T
//     (M128 N128 K64) into tensor memory, issued for key tile j+1 as soon
//     as the softmax has read S_q(j), then O_q += P_q V_j (M128 N64 K128) with
//     P_q read from tensor memory. Key tiles above the diagonal are never
//     issued. Each warpgroup has its own issuing thread, so neither waits on
//     the other's softmax.
//   * Warps 0-7 (softmax): two warpgroups. Warpgroup q serves query tile q of
//     the CTA's even items and tile 1 - q of its odd ones: tile i0 + 1 takes
//     one key tile more, and alternating it keeps one warpgroup from doing
//     every item's extra step while the other idles.
//     Each thread owns one query row (its TMEM lane) and all 128 columns of
//     every key tile: it loads the row of S from tensor memory, applies the
//     causal mask on the diagonal tile, runs the online softmax in base 2
//     (running max m, running sum l), rescales O in tensor memory when m
//     grows, and writes P as fp16. No row statistic crosses a thread. At the
//     end O is normalised and stored (bf16), and lse = ln2 * (m + log2 l).
//   * Warp 11 (convert): rewrites each V tile in shared memory from bf16 to
//     fp16 in place (or, in the FP8 forward, widens the e4m3 tile into a
//     separate fp16 tile), so that O += P V runs as an fp16 x fp16 product. P in
//     [0, 1] keeps 11 significant bits instead of 8, which matters on peaked
//     rows where one probability near 1 multiplies a large v. Every bf16 value
//     with |v| <= 65504 converts exactly (tiny ones to fp16 subnormals, within
//     3e-8); a v that is not finite with |v| <= 65504 is reported in the
//     status word.
//
// Tensor memory (512 columns x 128 lanes, fp32; index = warpgroup): S_0
// [0,128), S_1 [128,256), P_0 [256,320), P_1 [320,384) (fp16 pairs), O_0
// [384,448), O_1 [448,512).

#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace ga {
namespace fwd {

constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;       // issues for warpgroup 0, owns the TMEM allocation
constexpr int kMmaWarp1 = 10;     // issues for warpgroup 1
constexpr int kConvertWarp = 11;
// Register split (setmaxnreg): the TMA/MMA/convert warpgroup (warps 8-11) gives
// registers to the two softmax warpgroups, which hold a whole 128-column row
// of S. The total fits the block's launch allocation (kThreads x kLaunchRegs);
// the host refuses to launch if the kernel was compiled for fewer registers.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kRegsAux = 88;
constexpr uint32_t kRegsSoftmax = 208;
static_assert(128 * kRegsAux + 256 * kRegsSoftmax <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
static_assert(kProducerWarp == 8 && kConvertWarp == 11, "warps 8-11 form the aux warpgroup");
// The running max is raised only when a row's max grows by more than this many
// powers of two; until then P may reach 2^8 (well inside fp16).
constexpr float kRescaleLog2 = 8.f;
// One pair in kPolyEvery is exponentiated with the FMA-pipe polynomial.
constexpr int kPolyEvery = 6;
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint32_t col_s(int q) { return q * 128; }
__device__ __forceinline__ uint32_t col_p(int q) { return 256 + q * 64; }
__device__ __forceinline__ uint32_t col_o(int q) { return 384 + q * 64; }

// Bytes of one 128 x 64 Q or K tile: bf16, or e4m3 in the FP8 forward.
template <bool kFp8>
constexpr int kQKBytes = kFp8 ? kTileBytes / 2 : kTileBytes;

// The forward's item tables (ItemSchedule): the host fills them longest
// processing time first (items in decode_item order, heaviest first, each to
// the CTA with the least work so far) and splits a forward whose items do not
// fit the large one into several launches.
constexpr int kSchedSmall = 1024;
constexpr int kSchedMaxItems = 6144;

template <bool kFp8>
struct alignas(1024) Smem {
  uint8_t q[2][2][kQKBytes<kFp8>];   // [item slot][query tile]
  uint8_t k[kStages][kQKBytes<kFp8>];
  uint8_t v[kStages][kTileBytes];     // fp16 V as the P V product reads it
  uint8_t v8[kStages][kFp8 ? kTileBytes / 2 : 16];  // e4m3 V as loaded (FP8 only)
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages], v_ready[kStages];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
};

template <bool kFp8>
constexpr size_t kSmemBytes = sizeof(Smem<kFp8>) + 1024;  // + alignment slack

struct Item {
  int b, h, i0, has1, n_kv;
};

__device__ __forceinline__ Item decode_item(int k, const AttnShape& sh) {
  const int n_qt = ceil_div(sh.T, kBlockM);
  const int n_pairs = ceil_div(n_qt, 2);
  const int bh_count = sh.B * sh.H;
  const int p = n_pairs - 1 - k / bh_count;  // heaviest pairs first
  const int bh = k % bh_count;
  Item it;
  it.b = bh / sh.H;
  it.h = bh % sh.H;
  it.i0 = 2 * p;
  it.has1 = (2 * p + 1) < n_qt;
  it.n_kv = it.has1 ? 2 * p + 2 : 2 * p + 1;
  return it;
}

// The query tile of an item (0: i0, 1: i0 + 1) that warpgroup / issuer q
// serves in the CTA's it_cnt-th item. Tile i0 + 1 sees one key tile more, so
// the two swap on every other item: otherwise warpgroup 1 would take that
// extra step in every item and set the CTA's time alone.
__device__ __forceinline__ int item_tile(int q, uint32_t it_cnt) {
  return q ^ static_cast<int>(it_cnt & 1);
}

__host__ __device__ __forceinline__ int num_items(const AttnShape& sh) {
  return sh.B * sh.H * ceil_div(ceil_div(sh.T, kBlockM), 2);
}

// Epilogue of one query row: normalises its O (64 fp32 values read from
// tensor memory), stores it as bf16 and writes lse = ln2 * (m*c + log2 l).
// `c_log2` is the logits' scale in base 2 and `o_mul` a factor applied to O
// (1 for bf16 inputs; the V dequantisation for e4m3 inputs).
__device__ __forceinline__ void store_row(const uint32_t (&o)[64], int b, int h, int row, float m,
                                          float l, __nv_bfloat16* __restrict__ out,
                                          float* __restrict__ lse, const AttnShape& sh,
                                          float c_log2, float o_mul) {
  if (row >= sh.T) return;
  const float inv_l = o_mul / l;
  uint4* dst = reinterpret_cast<uint4*>(out + ((static_cast<size_t>(b) * sh.T + row) * sh.H + h) * kD);
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    uint4 w;
    w.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
    w.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
    w.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
    w.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
    dst[v] = w;
  }
  lse[(static_cast<size_t>(b) * sh.H + h) * sh.T + row] =
      (m * c_log2 + lg2(l)) * 0.69314718055994531f;
}

// kFp8 = false: qkv is bf16, map_qkv covers it (128-byte swizzle) and map_v8
// and dequant are unused. kFp8 = true: qkv holds e4m3 bytes; map_qkv covers
// it with the 64-byte swizzle (Q and K tiles), map_v8 without swizzle (V
// tiles, for the converter), and dequant[0..2] are the q, k, v dequantisation
// multipliers. S = Q K^T then multiplies e4m3 operands (kind::f8f6f4) and the
// softmax scale absorbs dequant[0] * dequant[1]; V becomes fp16 holding
// e4m3 * 2^-8 exactly, and O is multiplied by 2^8 * dequant[2] at the end.
// kV16: the v slot of qkv already holds fp16 (q and k stay bf16), as the
// c_attn GEMM writes it when asked; the convert warp then only passes each V
// tile on (kFp8 must be false).
template <bool kFp8, bool kV16, int kSchedItems>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap map_qkv,
                const __grid_constant__ CUtensorMap map_v8, __nv_bfloat16* __restrict__ out,
                float* __restrict__ lse, const AttnShape sh, const float* __restrict__ dequant,
                const __grid_constant__ ItemSchedule<kSchedItems> sched) {
  static_assert(!(kFp8 && kV16), "the FP8 forward widens its own e4m3 V");
  constexpr int kQK = kQKBytes<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  Smem<kFp8>& sm = *reinterpret_cast<Smem<kFp8>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = sh.H * kD;
  const int n_items = num_items(sh);
  volatile int* abort = &sm.abort;

  // This CTA's items, in order, and their count in the last slot (the
  // __syncthreads below publishes them to every role).
  __shared__ int items[kSchedSlots + 1];
  load_item_list(sched, items);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 2);   // one arrival per issuing thread
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 2);  // one arrival per query tile of the item
      mbar_init(&sm.v_ready[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&sm.s_full[q], 1);
      mbar_init(&sm.s_free[q], 4);   // the 4 softmax warps of the query tile
      mbar_init(&sm.p_full[q], 4);
      mbar_init(&sm.o_done[q], 1);
      mbar_init(&sm.drain[q], 1);
    }
    sm.abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&map_qkv);
    if (kFp8) tma_prefetch_desc(&map_v8);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp >= kProducerWarp) {
  regs_dealloc<kRegsAux>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA warp
    if (lane == 0) {
      uint32_t kv_it = 0, it_cnt = 0;
      for (int rnd = 0; rnd < items[kSchedSlots]; ++rnd) {
        const int k = items[rnd];
        if (k >= n_items) continue;
        const Item it = decode_item(k, sh);
        const int slot = it_cnt & 1;
        if (!mbar_wait(&sm.q_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteFwdProducer, abort)) break;
        mbar_arrive_expect_tx(&sm.q_full[slot], (it.has1 ? 2 : 1) * kQK);
        tma_load_3d(sm.q[slot][0], &map_qkv, &sm.q_full[slot], it.h * kD, it.i0 * kBlockM, it.b);
        if (it.has1)
          tma_load_3d(sm.q[slot][1], &map_qkv, &sm.q_full[slot], it.h * kD,
                      (it.i0 + 1) * kBlockM, it.b);
        ++it_cnt;
        bool ok = true;
        for (int j = 0; j < it.n_kv; ++j, ++kv_it) {
          const int s = kv_it % kStages;
          if (!mbar_wait(&sm.kv_empty[s], ((kv_it / kStages) & 1) ^ 1, kSiteFwdProducer, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kQK);
          tma_load_3d(sm.k[s], &map_qkv, &sm.kv_full[s], C + it.h * kD, j * kBlockN, it.b);
          if (kFp8)
            tma_load_3d(sm.v8[s], &map_v8, &sm.kv_full[s], 2 * C + it.h * kD, j * kBlockN, it.b);
          else
            tma_load_3d(sm.v[s], &map_qkv, &sm.kv_full[s], 2 * C + it.h * kD, j * kBlockN, it.b);
        }
        if (!ok) break;
      }
      // Drain: wait (bounded) for the last load issued into every buffer, so
      // no copy is still landing in shared memory when the CTA exits.
      for (int s = 0; s < kStages; ++s)
        if (kv_it > static_cast<uint32_t>(s))
          drain_wait(&sm.kv_full[s], ((kv_it - s + kStages - 1) / kStages - 1) & 1, kSiteFwdProducer);
      for (int s = 0; s < 2; ++s)
        if (it_cnt > static_cast<uint32_t>(s))
          drain_wait(&sm.q_full[s], ((it_cnt - s + 1) / 2 - 1) & 1, kSiteFwdProducer);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp1) {
    // ------------------------------------------------------------ MMA warps
    // One issuing thread per warpgroup q, for query tile item_tile(q, item)
    // of each item. Per item: S_q(0); then for each
    // key tile j the thread issues S_q(j+1) once the softmax has read S_q(j),
    // then O_q += P_q(j) V_j once P_q(j) is written and V_j converted.
    const int q = warp - kMmaWarp;
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_s8 = idesc_e4m3_f32(128, 128);
      constexpr uint32_t idesc_o = idesc_f16_f32(128, 64, 0, 1);
      const uint32_t t_s = tmem + col_s(q), t_p = tmem + col_p(q), t_o = tmem + col_o(q);
      uint32_t kv_it = 0, it_cnt = 0, s_cnt = 0, p_cnt = 0;
      bool ok = true;
      for (int rnd = 0; ok && rnd < items[kSchedSlots]; ++rnd) {
        const int k = items[rnd];
        if (k >= n_items) continue;
        const Item it = decode_item(k, sh);
        const int slot = it_cnt & 1;
        const int tq = item_tile(q, it_cnt);
        // Key tiles this query tile sees, and those the other one sees.
        const int n = tq == 0 ? it.i0 + 1 : (it.has1 ? it.i0 + 2 : 0);
        const int n_other = tq == 0 ? (it.has1 ? it.i0 + 2 : 0) : it.i0 + 1;
        if (n == 0) {
          // No second query tile in this item: this thread still releases its
          // share of the Q slot, after the slot's previous phase is complete
          // (an earlier arrival could complete that phase instead). It then
          // waits for the other issuer to release the slot too, i.e. for the
          // item to finish: every later wait of this thread is on a phase
          // parity, which is only unambiguous while the barrier is at most one
          // phase from the one expected. Skipping items without waiting let it
          // run ahead of the Q and K/V loads of the next item it serves and
          // read stale tiles.
          if (!mbar_wait(&sm.q_empty[slot], ((it_cnt >> 1) & 1) ^ 1, kSiteFwdMma, abort)) { ok = false; break; }
          mbar_arrive(&sm.q_empty[slot]);
          if (!mbar_wait(&sm.q_empty[slot], (it_cnt >> 1) & 1, kSiteFwdMma, abort)) { ok = false; break; }
        } else {
          if (!mbar_wait(&sm.q_full[slot], (it_cnt >> 1) & 1, kSiteFwdMma, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t qdesc = kFp8 ? smem_desc_sw64(smem_u32(sm.q[slot][tq]), 512)
                                      : smem_desc_sw128(smem_u32(sm.q[slot][tq]), 16, 1024);
          // S_q(jj) = Q_q K(jj)^T. bf16: K = 64 in four steps of 16 (32 bytes
          // each); e4m3: two steps of 32 (32 bytes each).
          auto issue_s = [&](int jj) -> bool {
            const uint32_t idx = kv_it + jj;
            const int st = idx % kStages;
            if (!mbar_wait(&sm.kv_full[st], (idx / kStages) & 1, kSiteFwdMma, abort)) return false;
            if (s_cnt > 0 && !mbar_wait(&sm.s_free[q], (s_cnt - 1) & 1, kSiteFwdMma, abort)) return false;
            tc_fence_after();
            if (kFp8) {
              const uint64_t kdesc = smem_desc_sw64(smem_u32(sm.k[st]), 512);
              mma_ss_f8(t_s, qdesc, kdesc, idesc_s8, 0u);
              mma_ss_f8(t_s, qdesc + 2, kdesc + 2, idesc_s8, 1u);
            } else {
              const uint64_t kdesc = smem_desc_sw128(smem_u32(sm.k[st]), 16, 1024);
              mma_ss(t_s, qdesc, kdesc, idesc_s, 0u);
#pragma unroll
              for (int kk = 1; kk < kD / 16; ++kk) mma_ss(t_s, qdesc + 2 * kk, kdesc + 2 * kk, idesc_s, 1u);
            }
            mma_commit(&sm.s_full[q]);
            ++s_cnt;
            return true;
          };
          if (!issue_s(0)) { ok = false; break; }
          for (int j = 0; j < n; ++j) {
            if (j + 1 < n && !issue_s(j + 1)) { ok = false; break; }
            const uint32_t idx = kv_it + j;
            const int st = idx % kStages;
            if (!mbar_wait(&sm.p_full[q], p_cnt & 1, kSiteFwdMma, abort)) { ok = false; break; }
            ++p_cnt;
            if (!mbar_wait(&sm.v_ready[st], (idx / kStages) & 1, kSiteFwdMma, abort)) { ok = false; break; }
            tc_fence_after();
            // 16 keys = 8 TMEM columns of P and 2048 bytes of V per step.
            const uint64_t vdesc = smem_desc_sw128(smem_u32(sm.v[st]), 128 * 128, 1024);
            mma_ts(t_o, t_p, vdesc, idesc_o, j > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < kBlockN / 16; ++kk)
              mma_ts(t_o, t_p + 8 * kk, vdesc + 128 * kk, idesc_o, 1u);
            mma_commit(&sm.o_done[q]);
            // The stage is released by two arrivals. A key tile the other query
            // tile does not see gets its second arrival here (its previous
            // phase is complete: this thread saw the tile land).
            mma_commit(&sm.kv_empty[st]);
            if (j >= n_other) mbar_arrive(&sm.kv_empty[st]);
          }
          if (!ok) break;
          mma_commit(&sm.q_empty[slot]);
        }
        kv_it += it.n_kv;
        ++it_cnt;
      }
      // Drain: every MMA this thread issued has finished before TMEM is freed.
      mma_commit(&sm.drain[q]);
      drain_wait(&sm.drain[q], 0, kSiteFwdMma);
    }
    __syncwarp();
  } else if (warp == kConvertWarp) {
    // ------------------------------------------------------------ convert V
    uint32_t kv_it = 0;
    bool ok = true;
    for (int rnd = 0; ok && rnd < items[kSchedSlots]; ++rnd) {
      const int k = items[rnd];
      if (k >= n_items) continue;
      const Item it = decode_item(k, sh);
      for (int j = 0; j < it.n_kv; ++j, ++kv_it) {
        const int s = kv_it % kStages;
        ok = mbar_wait(&sm.kv_full[s], (kv_it / kStages) & 1, kSiteFwdConvert, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (kFp8) {
          // e4m3 rows of 64 bytes, unswizzled, to fp16 rows of 128 bytes in
          // the 128-byte swizzle: the 16 e4m3 values of input chunk c of row
          // r fill fp16 chunks 2c and 2c + 1, stored at (chunk ^ (r & 7)).
#pragma unroll 2
          for (int idx = lane; idx < kTileBytes / 32; idx += 32) {
            const int rr = idx >> 2, c = idx & 3;
            const uint4 in = *reinterpret_cast<const uint4*>(sm.v8[s] + rr * 64 + c * 16);
            const uint4 lo = make_uint4(e4m3x2_to_f16x2_scaled(in.x, 0x4140u),
                                        e4m3x2_to_f16x2_scaled(in.x, 0x4342u),
                                        e4m3x2_to_f16x2_scaled(in.y, 0x4140u),
                                        e4m3x2_to_f16x2_scaled(in.y, 0x4342u));
            const uint4 hi = make_uint4(e4m3x2_to_f16x2_scaled(in.z, 0x4140u),
                                        e4m3x2_to_f16x2_scaled(in.z, 0x4342u),
                                        e4m3x2_to_f16x2_scaled(in.w, 0x4140u),
                                        e4m3x2_to_f16x2_scaled(in.w, 0x4342u));
            uint8_t* row = sm.v[s] + rr * 128;
            *reinterpret_cast<uint4*>(row + (((2 * c) ^ (rr & 7)) << 4)) = lo;
            *reinterpret_cast<uint4*>(row + (((2 * c + 1) ^ (rr & 7)) << 4)) = hi;
          }
        } else if (!kV16) {
          uint4* tile = reinterpret_cast<uint4*>(sm.v[s]);
          // Running max of |v| over the converted fp16 values: a bf16 beyond
          // fp16's range rounds to inf, so inf or NaN here flags the tile.
          uint32_t mag = 0;
#pragma unroll 4
          for (int c = lane; c < kTileBytes / 16; c += 32) {
            uint4 w = tile[c];
            uint32_t* u = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              // bf16 -> fp32 is exact (a shift); fp32 -> fp16 rounds to
              // nearest, exact for every bf16 value with |v| <= 65504 except
              // fp16 subnormals (|v| < 6.1e-5, within 3e-8).
              u[e] = pack_f16(__uint_as_float(u[e] << 16), __uint_as_float(u[e] & 0xFFFF0000u));
              mag = max_abs_f16x2(mag, u[e]);
            }
            tile[c] = w;
          }
          if ((mag & 0x7FFFu) >= kF16InfBits || ((mag >> 16) & 0x7FFFu) >= kF16InfBits)
            record_failure(kFwdValueRange);
        }
        // Generic-proxy stores must be visible to the tensor core (async proxy).
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.v_ready[s]);
      }
    }
  }
  } else {
    regs_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    // The logits' scale in base 2, and the factor O is multiplied with at the
    // end (both fold in the dequantisation of e4m3 inputs).
    const float c_log2 = kFp8 ? sh.scale_log2 * dequant[0] * dequant[1] : sh.scale_log2;
    const float o_mul = kFp8 ? 256.f * dequant[2] : 1.f;
    const int q = warp >> 2;                       // warpgroup; its query tile is item_tile()
    const int r = ((warp & 3) << 5) + lane;        // row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t t_s = tmem + lane_base + col_s(q);
    const uint32_t t_p = tmem + lane_base + col_p(q);
    const uint32_t t_o = tmem + lane_base + col_o(q);
    uint32_t s_cnt = 0, o_cnt = 0;
    // The finished item whose O still sits in tensor memory. It is read out
    // while the next item's first tile is processed, just before that tile's
    // P goes to tensor memory (the next P V product then overwrites O); the
    // normalisation and stores follow once that tile is handed over.
    bool pending = false;
    int p_b = 0, p_h = 0, p_row = 0;
    float p_m = 0.f, p_l = 0.f;
    bool ok = true;
    uint32_t it_cnt = 0;
    for (int rnd = 0; ok && rnd < items[kSchedSlots]; ++rnd) {
      const int k = items[rnd];
      if (k >= n_items) continue;
      const Item it = decode_item(k, sh);
      const int tq = item_tile(q, it_cnt++);
      if (tq == 1 && !it.has1) continue;
      const int i = it.i0 + tq;
      const int row = i * kBlockM + r;
      // Running max m (raw logit units, as read from S) and running sum l of
      // 2^(s*c - m*c), c = c_log2. m is only raised when the row max
      // grows by more than kRescaleLog2 in log2 units; until then P and l keep
      // using the stale m, which stays exact because O / l uses the same m.
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j <= i; ++j) {
        ok = mbar_wait(&sm.s_full[q], s_cnt & 1, kSiteFwdSoftmax, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        float x[128];
        {
          uint32_t* u = reinterpret_cast<uint32_t*>(x);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(t_s + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * c));
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[q]);

        if (j == i) {
          const int lim = row - j * kBlockN;  // columns c > lim are future keys
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (c > lim) ? -INFINITY : x[c];
        }
        // Row max: 8 independent chains of 3-input max.
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmax3(x[e], x[8 + e], x[16 + e]);
#pragma unroll
        for (int c = 24; c < 120; c += 16) {
#pragma unroll
          for (int e = 0; e < 8; ++e) mx8[e] = fmax3(mx8[e], x[c + e], x[c + 8 + e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], x[120 + e]);
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const bool grow = (mx - m) * c_log2 > kRescaleLog2;  // always true on j == 0
        const float m_new = grow ? mx : m;
        const float alpha = grow ? ex2((m - m_new) * c_log2) : 1.f;
        const float neg_mc = -m_new * c_log2;
        const bool flush = (j == 0) && pending;
        // The FP8 forward keeps two more values live through the loop below
        // (the runtime logit scale and output factor), so it waits for the
        // previous P V product first and stores each half of P as soon as it
        // is packed, holding 32 packed registers instead of 64.
        constexpr bool kEarlyWait = kFp8;
        if (kEarlyWait && (j > 0 || flush)) {
          ok = mbar_wait(&sm.o_done[q], o_cnt & 1, kSiteFwdSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++o_cnt;
          tc_fence_after();
        }
        // p = 2^(s*c - m*c), row sum, and fp16 packing of P in one pass. Every
        // kPolyEvery-th pair is exponentiated on the FMA pipe (exp2_poly2), the
        // rest on the exp unit, whose 16/clk rate bounds this loop otherwise.
        uint32_t pk[64];
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c2 = 0; c2 < 64; ++c2) {
          float y0, y1, p0, p1;
          fma2(x[2 * c2], x[2 * c2 + 1], c_log2, neg_mc, y0, y1);
          if (c2 % kPolyEvery == kPolyEvery - 1) {
            exp2_poly2(y0, y1, p0, p1);
          } else {
            p0 = ex2(y0);
            p1 = ex2(y1);
          }
          add2(sa[c2 & 3], sb[c2 & 3], p0, p1);
          pk[c2] = pack_f16_nonneg(p0, p1);
          if (kEarlyWait && c2 == 31) tmem_st32(t_p, *reinterpret_cast<uint32_t(*)[32]>(pk));
        }
        const float sum = ((sa[0] + sb[0]) + (sa[1] + sb[1])) + ((sa[2] + sb[2]) + (sa[3] + sb[3]));
        l = l * alpha + sum;
        m = m_new;

        if (!kEarlyWait && (j > 0 || flush)) {
          // O must hold P_{j-1} V_{j-1} (or the finished item's last product)
          // before it is rescaled or read, and before P is reused.
          ok = mbar_wait(&sm.o_done[q], o_cnt & 1, kSiteFwdSoftmax, abort);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++o_cnt;
          tc_fence_after();
        }
        if (!kEarlyWait) tmem_st32(t_p, *reinterpret_cast<uint32_t(*)[32]>(pk));
        tmem_st32(t_p + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        if (flush) {
          // The finished item's O is read before this tile's P V product (which
          // starts only after the arrival below) overwrites it.
          uint32_t o[64];
          tmem_ld32(t_o, *reinterpret_cast<uint32_t(*)[32]>(o));
          tmem_ld32(t_o + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
          tmem_wait_ld();
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[q]);
          store_row(o, p_b, p_h, p_row, p_m, p_l, out, lse, sh, c_log2, o_mul);
          pending = false;
        } else {
          if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t oo[32];
              tmem_ld32(t_o + 32 * c, oo);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) oo[e] = __float_as_uint(__uint_as_float(oo[e]) * alpha);
              tmem_st32(t_o + 32 * c, oo);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[q]);
        }
      }
      if (!ok) break;
      pending = true;
      p_b = it.b;
      p_h = it.h;
      p_row = row;
      p_m = m;
      p_l = l;
    }
    if (ok && pending) {
      ok = mbar_wait(&sm.o_done[q], o_cnt & 1, kSiteFwdSoftmax, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        ++o_cnt;
        tc_fence_after();
        uint32_t o[64];
        tmem_ld32(t_o, *reinterpret_cast<uint32_t(*)[32]>(o));
        tmem_ld32(t_o + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
        tmem_wait_ld();
        tc_fence_before();
        store_row(o, p_b, p_h, p_row, p_m, p_l, out, lse, sh, c_log2, o_mul);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd
}  // namespace ga
