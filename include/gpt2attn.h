/*
 * gpt2attn.h: C ABI of the fused causal self-attention library (sm_100a).
 *
 * The operation is the attention step of every GPT-2 (124M) block: causal
 * multi-head self-attention on the packed q,k,v activations, computed the
 * "flash attention" way, without ever storing the T x T attention matrix
 * ("Let's reproduce GPT-2 (124M)" video summary page, glossary table, row
 * "flash attention"; "Andrej Karpathy - Lets reproduce GPT 2 124M" video
 * description, chapter 02:00:18 "flash attention"). The model is 12 layers of
 * width C = 768 (video summary page, closing summary paragraph), i.e. H = 12
 * heads of D = 64.
 *
 * Definition (per batch b, head h; i = query row, j = key row):
 *     s_ij  = scale * q_i . k_j  for j <= i (key j visible iff j <= i)
 *     lse_i = ln sum_{j<=i} exp(s_ij)
 *     P_ij  = exp(s_ij - lse_i),   out_i = sum_j P_ij v_j
 * and its gradients dq, dk, dv for an upstream gradient dout.
 *
 * Layouts (all row-major, contiguous, device memory):
 *     qkv   bf16 (B, T, 3, H, D)  the GPT-2 c_attn output (B, T, 3C) split into
 *                                 q (slot 0), k (slot 1), v (slot 2), head-major
 *     out   bf16 (B, T, H, D)     = (B, T, C), ready for c_proj
 *     lse   fp32 (B, H, T)        natural log of the scaled logits' sum of exp
 *     dout  bf16 (B, T, H, D)
 *     dqkv  bf16 (B, T, 3, H, D)  overwritten: slot 0 = dq, 1 = dk, 2 = dv
 *
 * Conventions:
 *   - Only D == 64 is supported (GA_ERR_UNSUPPORTED otherwise).
 *   - B, T, H >= 1; B*T*3*H*D must be below 2^31 elements.
 *   - Every pointer must be non-null and 16-byte aligned.
 *   - scale must be finite and > 0; GPT-2 uses 1/sqrt(D) = 0.125.
 *   - The caller owns every buffer, including the backward workspace. The
 *     library allocates nothing per call. Between calls it keeps only host
 *     caches (per-device set-up and the TMA descriptors of recently seen
 *     tensors, keyed by address, extents and layout, each behind a mutex) and
 *     a device status word that records a timed-out wait.
 *   - Calls only enqueue work on `stream` (the legacy default stream when
 *     NULL). They never synchronise. Arguments are checked before anything is
 *     launched: on any error nothing is launched and the status says why.
 *   - Inputs and outputs must not overlap.
 *   - No dropout, no attention bias, and no non-causal mode.
 */
#ifndef GPT2ATTN_H_
#define GPT2ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that this header
 * needs no CUDA header. */
typedef struct CUstream_st* gpt2attn_stream_t;

typedef enum {
  GA_OK = 0,
  GA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad scale, size overflow */
  GA_ERR_UNSUPPORTED = 2, /* a shape the kernels do not implement (D != 64) */
  GA_ERR_ALIGNMENT = 3,   /* a pointer that is not 16-byte aligned */
  GA_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the query result */
  GA_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
  GA_ERR_TIMEOUT = 6,     /* a device-side wait gave up (see gpt2_attn_last_device_status) */
  GA_ERR_RANGE = 7        /* the forward met a v entry outside the fp16 range (|v| > 65504, inf or NaN) */
} ga_status;

/*
 * Forward: out and lse from qkv.
 *   qkv   [in]  bf16 (B,T,3,H,D), device
 *   out   [out] bf16 (B,T,H,D), device, fully overwritten
 *   lse   [out] fp32 (B,H,T), device, fully overwritten
 * Steps on the device: tiles of 128 queries stream 128-key tiles of K and V
 * through shared memory (TMA), S = Q K^T and O += P V run on the tensor cores
 * with fp32 accumulators in tensor memory, the online softmax runs in
 * registers, key tiles above the diagonal are skipped, and lse is written
 * per query row. S = Q K^T multiplies bf16 operands. O += P V multiplies
 * fp16 operands: P keeps 11 significant bits, and each bf16 v with
 * 2^-14 <= |v| <= 65280 converts to fp16 exactly (smaller ones move by less
 * than 2^-15). A v entry beyond fp16's range (|v| >= 65536, inf or NaN) is
 * reported as GA_ERR_RANGE by gpt2_attn_last_device_status; the outputs of
 * that call are then undefined.
 * The work items (one (b,h) and a pair of query tiles each) are dealt to a
 * persistent grid of at most one CTA per SM by the host, longest processing
 * time first (gpt2_attn_fwd_item_schedule returns the deal); the deal is
 * cached per shape. A forward of more than 6144 items is split into several
 * launches on `stream`. The deal never changes the result.
 */
ga_status gpt2_attn_fwd(const void* qkv, void* out, float* lse,
                        int B, int T, int H, int D, float scale,
                        gpt2attn_stream_t stream);

/*
 * gpt2_attn_fwd for a qkv whose v slot already holds fp16 (q and k bf16), as
 * gpt2_attn_qkv_proj_v16 writes it: the same computation and outputs, without
 * the in-kernel bf16 -> fp16 conversion of each V tile (the P V product runs
 * in fp16 either way). For a v that bf16 and fp16 both hold exactly, out and
 * lse are bit-identical to gpt2_attn_fwd's on the bf16 qkv. For inference
 * and prefill: the backward reads v as bf16. Same arguments, layout and
 * errors as gpt2_attn_fwd, except that no v range check is needed (no
 * GA_ERR_RANGE).
 */
ga_status gpt2_attn_fwd_v16(const void* qkv, void* out, float* lse, int B, int T, int H, int D,
                            float scale, gpt2attn_stream_t stream);

/*
 * Size in bytes of the workspace gpt2_attn_bwd needs for this shape:
 * Delta, fp32 (B,H,T), at offset 0, rounded up to 256 bytes, where
 * Delta[b,h,t] = sum_d dout[b,t,h,d] * out[b,t,h,d]. After a gpt2_attn_bwd
 * call it holds that call's Delta.
 */
ga_status gpt2_attn_bwd_workspace_size(int B, int T, int H, int D, size_t* bytes);

/*
 * Backward: dqkv from qkv, out, dout and lse (out and lse as written by
 * gpt2_attn_fwd for the same qkv and scale).
 *   qkv, out, dout, lse [in]
 *   dqkv      [out] bf16 (B,T,3,H,D), fully overwritten (not accumulated)
 *   workspace [scratch] device, >= gpt2_attn_bwd_workspace_size bytes,
 *             16-byte aligned, owned by the caller, must not be shared by
 *             calls that run concurrently
 * Two launches on `stream` (the split backward below): dq per query tile,
 * which also computes that tile's Delta, recomputes P from lse and
 * accumulates dq in tensor memory with no atomics; then dk and dv per key
 * tile, which read Delta and recompute P. The result is bitwise
 * deterministic.
 */
ga_status gpt2_attn_bwd(const void* qkv, const void* out, const void* dout,
                        const float* lse, void* dqkv,
                        void* workspace, size_t workspace_bytes,
                        int B, int T, int H, int D, float scale,
                        gpt2attn_stream_t stream);

/*
 * The two steps of gpt2_attn_bwd as separate calls, with the same argument
 * conventions. gpt2_attn_bwd is exactly gpt2_attn_bwd_dq followed by
 * gpt2_attn_bwd_dkdv on one stream. `delta` is fp32 (B,H,T), caller-owned,
 * 16-byte aligned, where delta[b,h,t] = sum_d dout[b,t,h,d] * out[b,t,h,d]
 * (the row term sum_j P_ij dP_ij of the softmax Jacobian).
 *
 * gpt2_attn_bwd_dq: writes dqkv slot 0 (dq) and delta [out]; dqkv slots 1
 *   and 2 untouched. One CTA per 128-query tile computes the tile's delta
 *   from its dout and out rows, recomputes P and dP for every key tile at or
 *   before it and accumulates dq in tensor memory (no atomics).
 * gpt2_attn_bwd_dkdv: writes dqkv slots 1 (dk) and 2 (dv); slot 0 untouched.
 *   Reads delta [in] (as written by gpt2_attn_bwd_dq or
 *   gpt2_attn_bwd_preprocess). One CTA per 128-key tile recomputes P from
 *   lse for every query tile at or after it and accumulates dk, dv in tensor
 *   memory.
 * gpt2_attn_bwd_preprocess: delta alone, in its own memory-bound launch
 *   (for callers that need delta without dq).
 */
ga_status gpt2_attn_bwd_dq(const void* qkv, const void* out, const void* dout,
                           const float* lse, float* delta, void* dqkv,
                           int B, int T, int H, int D, float scale,
                           gpt2attn_stream_t stream);
ga_status gpt2_attn_bwd_dkdv(const void* qkv, const void* dout, const float* lse,
                             const float* delta, void* dqkv,
                             int B, int T, int H, int D, float scale,
                             gpt2attn_stream_t stream);
ga_status gpt2_attn_bwd_preprocess(const void* out, const void* dout, float* delta,
                                   int B, int T, int H, int D, gpt2attn_stream_t stream);

/*
 * The fused backward: the same dqkv from one pass over the causal tiles
 * (S, P, dP, dS computed once per tile instead of twice), bitwise
 * deterministic. On B200 at GPT-2 shapes it is slower than gpt2_attn_bwd:
 * the ordered dq reduction across CTAs costs more than the recompute it
 * saves. It needs a larger workspace, with n = ceil(T/128):
 * 4*B*H*T + 4*B*H*(128n)*D + 4*B*H*n bytes, each part rounded up to 256.
 * Layout, byte offsets:
 *   0                          Delta fp32 (B,H,T)
 *   align256(4*B*H*T)          dq partial sums, fp32, per 128-row query tile
 *   + align256(4*B*H*128n*D)   dq ordering counters, uint32 (B,H,n)
 *
 * gpt2_attn_bwd_fused_workspace_size: that size.
 * gpt2_attn_bwd_prepare: Delta into the workspace, and zeroes its counters.
 *   GA_ERR_WORKSPACE if the workspace is missing or too small.
 * gpt2_attn_bwd_fused: needs a workspace prepared by gpt2_attn_bwd_prepare
 *   for the same out, dout and shape (earlier on the same stream). One CTA
 *   per 128-key tile j recomputes P from lse for every query tile i >= j
 *   (from the last to the diagonal one) and issues dV += P^T dO and
 *   dK += dS^T Q (kept in tensor memory) and dQ_ij = dS K_j. Each dQ_ij is
 *   added to the workspace's fp32 sum for query tile i in ascending j (key
 *   tile j waits until tiles 0..j-1 have added); key tile i adds last and
 *   writes dq = scale * sum as bf16. Writes all three dqkv slots.
 */
ga_status gpt2_attn_bwd_fused_workspace_size(int B, int T, int H, int D, size_t* bytes);
ga_status gpt2_attn_bwd_prepare(const void* out, const void* dout, void* workspace,
                                size_t workspace_bytes, int B, int T, int H, int D,
                                gpt2attn_stream_t stream);
ga_status gpt2_attn_bwd_fused(const void* qkv, const void* dout, const float* lse,
                              void* workspace, size_t workspace_bytes, void* dqkv,
                              int B, int T, int H, int D, float scale,
                              gpt2attn_stream_t stream);

/*
 * Decode attention: the attention output of query row t alone, over the keys
 * and values of rows 0..t of the same packed qkv buffer (the newest token of a
 * generation step, with the earlier rows' k and v kept in the buffer). This is
 * row t of gpt2_attn_fwd's result, computed without the other rows.
 *   qkv   [in]  bf16 (B,T,3,H,D), device; rows 0..t are read (q only of row t)
 *   t     [in]  0 <= t < T
 *   out   [out] bf16 (B,H,D), device
 *   lse   [out] fp32 (B,H), device: natural log of sum_j exp(scale q.k_j)
 *   workspace [scratch] >= gpt2_attn_decode_workspace_size bytes, 16-byte
 *         aligned, not shared by calls that run concurrently
 * Two launches on `stream`: per 128-key chunk of each (b,h), partial max, sum
 * and unnormalised output (the chunk's k and v rows staged in shared memory
 * by TMA; fp32 on the CUDA cores: the step is bound by reading k and v); then
 * one combine per (b,h). GA_ERR_INVALID_ARG for t outside
 * [0, T) or B, H above 65535.
 */
ga_status gpt2_attn_decode_workspace_size(int B, int T, int H, int D, size_t* bytes);
ga_status gpt2_attn_decode(const void* qkv, int t, void* out, float* lse,
                           void* workspace, size_t workspace_bytes,
                           int B, int T, int H, int D, float scale,
                           gpt2attn_stream_t stream);

/*
 * gpt2_attn_bwd without a workspace argument, for callers that cannot
 * allocate device memory: a plugin that is handed only its input and output
 * buffers by a host application that owns all device memory, or a program
 * that reserves the GPU's memory at start-up and may not call cudaMalloc (or
 * pay for its implicit synchronisation) afterwards. The pages have no
 * counterpart to this entry point; it exists for such callers only.
 *   Same arguments, layouts and results as gpt2_attn_bwd. Delta is kept in a
 *   fixed array in the library's static device memory instead of a caller
 *   workspace: 2^20 floats (4 MiB) on every GPU that loads the library, held
 *   until the process exits. Shapes with B*H*T > 1,048,576 are rejected with
 *   GA_ERR_WORKSPACE before anything is launched.
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.
 *   Every call shares the array and leaves its own Delta in it. Each call
 *   rewrites all the Delta values it reads, so nothing needs clearing; but
 *   calls that overlap on the GPU (other streams, other host threads on the
 *   same device) race on the array and must be serialised by the caller.
 */
ga_status gpt2_attn_bwd_noalloc(const void* qkv, const void* out, const void* dout,
                                const float* lse, void* dqkv,
                                int B, int T, int H, int D, float scale,
                                gpt2attn_stream_t stream);

/*
 * FP8 forward: the attention of e4m3 q, k, v with one scale per tensor. The
 * llm.c page plans FP8 training ("Réimplémenter à bas coût le modèle GPT-2
 * avec llm.c", FAQ entry on FP8); the pages fix no format, so each of q, k
 * and v gets the scale that maps its largest magnitude to 448, the largest
 * e4m3 value. Results are those of the attention of the dequantised inputs
 * (e4m3 value * dequant), not of the bf16 ones: the e4m3 rounding of the
 * inputs moves the output far more than the bf16 path's error.
 *
 * gpt2_attn_fp8_quantize: qkv (bf16, as gpt2_attn_fwd reads it) to
 *   qkv8  [out] e4m3 bytes (B,T,3,H,D), same layout, one byte per element
 *   scales [out/scratch] fp32[8], device, 16-byte aligned: [0..2] receive the
 *          dequantisation multipliers of q, k, v (amax / 448, or 1 for an
 *          all-zero tensor); [4..6] are scratch (the amax words)
 *   with amax = max |x| per slot, x8 = e4m3(x * (448 / amax)) rounded to
 *   nearest even (every fp32 step correctly rounded). Three launches on
 *   `stream`: clear the amax words, reduce amax, scale and round. NaN inputs
 *   are skipped by the amax and stay NaN.
 * gpt2_attn_fwd_fp8: out and lse from qkv8 and scales as written by
 *   gpt2_attn_fp8_quantize (earlier on the same stream); out, lse and scale
 *   as for gpt2_attn_fwd. S = Q K^T multiplies the e4m3 operands on the
 *   tensor cores (kind::f8f6f4, fp32 accumulation); the softmax scale absorbs
 *   dequant_q * dequant_k; V is widened to fp16 (exact) for O += P V, and O is
 *   multiplied by dequant_v.
 */
ga_status gpt2_attn_fp8_quantize(const void* qkv, void* qkv8, float* scales,
                                 int B, int T, int H, int D, gpt2attn_stream_t stream);
ga_status gpt2_attn_fwd_fp8(const void* qkv8, const float* scales, void* out, float* lse,
                            int B, int T, int H, int D, float scale,
                            gpt2attn_stream_t stream);

/*
 * The two dense layers on either side of attention in a GPT-2 block
 * ("Andrej Karpathy - Lets reproduce GPT 2 124M" video description, chapter
 * 00:13:47, the GPT-2 nn.Module; "Comment recréer GPT2 en 4 heures ?",
 * section 5, the rearranged blocks), on the tensor cores (bf16 inputs, fp32
 * accumulation in tensor memory, bias added in fp32, one rounding to bf16).
 * Weights use nn.Linear's layout (out_features, in_features), row-major.
 * C = H * D with D == 64; B, T, H as for the attention calls; every pointer
 * 16-byte aligned; B*T*3C below 2^31.
 *
 * gpt2_attn_qkv_proj (c_attn): qkv = x W_attn^T + b_attn
 *   x      [in]  bf16 (B,T,C)
 *   w_attn [in]  bf16 (3C, C)
 *   b_attn [in]  bf16 (3C)
 *   qkv    [out] bf16 (B,T,3,H,D): the row-major (B*T, 3C) result, which is
 *                exactly the packed layout gpt2_attn_fwd reads
 * gpt2_attn_out_proj (c_proj): y = out W_proj^T + b_proj
 *   out    [in]  bf16 (B,T,H,D): gpt2_attn_fwd's output, read as (B*T, C)
 *   w_proj [in]  bf16 (C, C)
 *   b_proj [in]  bf16 (C)
 *   y      [out] bf16 (B,T,C)
 * One launch each on `stream`; inputs and outputs must not overlap.
 */
ga_status gpt2_attn_qkv_proj(const void* x, const void* w_attn, const void* b_attn,
                             void* qkv, int B, int T, int H, int D,
                             gpt2attn_stream_t stream);
/*
 * As gpt2_attn_qkv_proj, but the v slot of qkv (columns [2C, 3C)) is written
 * in fp16 (round to nearest; |v| above 65504 becomes inf), q and k in bf16:
 * the input gpt2_attn_fwd_v16 reads. A qkv written this way is not an input
 * of gpt2_attn_fwd or of the backward, which read v as bf16.
 */
ga_status gpt2_attn_qkv_proj_v16(const void* x, const void* w_attn, const void* b_attn,
                                 void* qkv, int B, int T, int H, int D,
                                 gpt2attn_stream_t stream);
ga_status gpt2_attn_out_proj(const void* out, const void* w_proj, const void* b_proj,
                             void* y, int B, int T, int H, int D,
                             gpt2attn_stream_t stream);

/*
 * Self-test of the device-side failure path that every kernel of this library
 * shares. Launches one small kernel on `stream` in which one thread waits on
 * a shared-memory barrier that nothing ever completes, bounded by
 * `limit_ns` nanoseconds (0 < limit_ns <= 1e9, else GA_ERR_INVALID_ARG).
 * When the limit passes, that thread records its wait site (0x501) in the
 * device status word and raises the block's abort flag; a second waiter on
 * the same barrier, bounded by the library's usual 2 s limit, sees the flag
 * and returns without recording, and the block frees its tensor memory and
 * exits. Nothing traps or faults, and the context stays usable.
 * A following gpt2_attn_last_device_status returns GA_ERR_TIMEOUT with
 * detail >> 32 == 0x501 (and clears the word). This is the same bounded wait
 * the attention kernels use; this entry point exists so that the path that
 * ends it can be exercised on purpose. It has no counterpart on the pages.
 */
ga_status gpt2_attn_selftest_wait_timeout(unsigned long long limit_ns,
                                          gpt2attn_stream_t stream);

/*
 * The forward's deal of work items to CTAs and launches, as gpt2_attn_fwd,
 * _fwd_v16 and _fwd_fp8 make it for (B, T, H) on a device with num_sms SMs.
 * An item is one (b, h) and a pair of adjacent 128-row query tiles; there are
 * n_items = B*H*ceil(ceil(T/128)/2) of them, numbered heaviest first (item k
 * covers query tiles 2p and 2p + 1, p = ceil(ceil(T/128)/2) - 1 - k / (B*H),
 * of head (b, h) = divmod(k % (B*H), H)). The items are split into launches
 * of consecutive items (one launch unless they exceed one kernel parameter
 * table: 6144 items, 64 per CTA), each on min(its items, num_sms, 160) CTAs.
 * Within a launch every item goes, in order, to the CTA with the least work
 * so far (longest processing time first; an item of n key tiles counts
 * n + 2.5 tile steps). For every item k, launch[k] receives its launch,
 * cta[k] the CTA that runs it and pos[k] its place in that CTA's list (a CTA
 * runs its items in increasing pos). `n` is the capacity of the three arrays
 * (>= n_items). Returns the number of launches, or -GA_ERR_INVALID_ARG on a
 * null pointer, a non-positive size or n < n_items. Host code only: no CUDA
 * call, usable without a GPU. The deal changes which CTA computes an item,
 * never what it computes.
 */
int gpt2_attn_fwd_item_schedule(int B, int T, int H, int num_sms, int* launch, int* cta,
                                int* pos, long n);

/*
 * Synchronises `stream`, then reads and clears the device status word.
 * Returns GA_ERR_TIMEOUT if a kernel of this library gave up on a device-side
 * wait since the last call (the kernel then stopped early and its outputs are
 * undefined), GA_ERR_RANGE if the forward met a v entry outside the fp16
 * range, GA_ERR_CUDA if the synchronisation itself failed, GA_OK otherwise.
 * If `detail` is non-null it receives the raw status word (0 when clean;
 * otherwise the high 32 bits name the kernel and wait site and the low 32
 * bits the block index).
 */
ga_status gpt2_attn_last_device_status(gpt2attn_stream_t stream, unsigned long long* detail);

/*
 * The CUDA failure behind the latest GA_ERR_CUDA returned by any entry point
 * of this library (from any host thread), then cleared; 0 if none since the
 * last read. High 32 bits: the failing step (1 device set-up, 2 TMA
 * descriptor encoding, 3 kernel launch); low 32 bits: its cudaError_t (steps
 * 1 and 3; 0 when a non-CUDA set-up check failed) or CUresult (step 2).
 */
unsigned long long gpt2_attn_last_cuda_error(void);

/* Static, human-readable name of a status code. Never returns NULL. */
const char* gpt2_attn_status_string(ga_status s);

/* Library version as 10000*major + 100*minor + patch. */
int gpt2_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GPT2ATTN_H_ */
