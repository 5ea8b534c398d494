/*
 * spa.h -- block-sparse long-context attention prefill on B200 (sm_100a).
 *
 * Two stages, both running entirely on the GPU:
 *
 *   sparse_prefill_plan   picks, for every 128-row query block, which keys
 *                         outside the always-kept sink and local windows are
 *                         attended to, and writes them as ascending index
 *                         lists into a caller-owned workspace;
 *   sparse_prefill_attn   runs causal softmax attention over exactly those
 *                         keys (sink + selected + local) and writes O and,
 *                         optionally, the row log-sum-exp.
 *
 * Selection modes
 *   SPA_MODE_ANCHOR  AnchorAttention: Difference-Aware Sparse Attention with
 *                    Stripe Granularity, Eq. (1)-(3): anchor x_a[i] = max score
 *                    over the sink and local keys of row i; candidate key j of
 *                    block b is kept iff mean_i(x_a[i]) - mean_i(q_i).k_j*scale
 *                    <= theta (key-stripe granularity, block_k = 1).
 *   SPA_MODE_SALE    SALE: Low-bit Estimation for Efficient Sparse Attention in
 *                    Long-context LLM Prefilling, Sec. 3.2-3.4: S~ from 4-bit
 *                    quantised Q and smoothed K; key block kb (block_k keys) is
 *                    kept iff some row i and key j in kb have
 *                    S~_ij >= ln(tau * el_i) + em_i, em/el being the max and the
 *                    sum of exp(S~ - em) over the row's sink and local keys.
 *   SPA_MODE_DENSE   no selection: every causal key (the "same kernel, dense"
 *                    reference point for speedups).
 *
 * Geometry (all modes).  Query block b = rows [b*block_q, (b+1)*block_q) (the
 * last one may be ragged).  Sink keys [0, sink).  Local window
 * [ls_b, (b+1)*block_q), ls_b = max(0, (b+1)*block_q - local), causally cut
 * per row.  Candidates C_b = [sink, ls_b).  Row i of block b attends to
 * (sink u local u selected(b)) n {j <= i}.
 *
 * Tensors.  Q: bf16 [B, Hq, L, 128]; K, V: bf16 [B, Hkv, L, 128]; O: bf16
 * [B, Hq, L, 128]; LSE: fp32 [B, Hq, L] (natural log).  Row-major, head_dim
 * innermost, contiguous, device pointers, 16-byte aligned.  q head h reads kv
 * head h / (Hq / Hkv) (grouped-query attention).
 *
 * Ownership.  The caller allocates and owns Q, K, V, O, LSE and the
 * workspace; the library never allocates or frees device memory and keeps no
 * state between calls.  Every call is asynchronous on the given stream except
 * sparse_prefill_stats, which synchronises that stream.  A workspace written
 * by sparse_prefill_plan stays valid for sparse_prefill_attn and
 * sparse_prefill_stats until the next plan on the same workspace.  Two calls
 * that share a workspace must not overlap on the GPU.
 *
 * Errors.  Argument, shape, alignment and workspace-size errors are returned
 * synchronously, before anything is launched.  A failed launch returns
 * SPA_ERR_CUDA.  Kernels never trap: a bounded wait that expires, or an index
 * that fails a device-side check, sets a bit in the workspace error word and
 * the kernel returns early; sparse_prefill_stats reports it (as
 * SPA_ERR_TIMEOUT or SPA_ERR_INVALID) and the outputs of that call are
 * undefined.
 */
#ifndef SPA_H_
#define SPA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define SPA_API __attribute__((visibility("default")))
#else
#define SPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPA_OK = 0,
  SPA_ERR_INVALID = 1,      /* bad argument (null/misaligned pointer, bad size or value) */
  SPA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (head_dim != 128, causal == 0, ...) */
  SPA_ERR_WORKSPACE = 3,    /* workspace smaller than sparse_prefill_workspace_bytes() */
  SPA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  SPA_ERR_TIMEOUT = 5       /* a device-side bounded wait expired (reported by stats) */
} spa_status;

typedef enum {
  SPA_MODE_ANCHOR = 0,
  SPA_MODE_SALE = 1,
  SPA_MODE_DENSE = 2
} spa_mode;

typedef struct {
  int32_t batch;          /* B >= 0 (0 -> every call is a no-op) */
  int32_t heads_q;        /* Hq >= 1 */
  int32_t heads_kv;       /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t seq_len;        /* L >= 0; B*max(Hq,Hkv)*L < 2^31 */
  int32_t head_dim;       /* must be 128 */
  int32_t causal;         /* must be 1 */
  int32_t block_q;        /* must be 128 */
  int32_t block_k;        /* ANCHOR: 1 (key stripes); SALE: 16, 32, 64 or 128; DENSE: ignored */
  int32_t sink;           /* >= 0; SALE: multiple of block_k */
  int32_t local;          /* >= block_q, multiple of block_q */
  int32_t step;           /* >= 1: query blocks grouped per selection (AnchorAttention's
                             step); a candidate kept by any block of a group of `step`
                             consecutive blocks is kept by all of them, within each
                             block's own candidate range.  1 = each block for itself */
  spa_mode mode;
  float theta;            /* ANCHOR threshold, scaled-logit units; +inf keeps all; NaN invalid */
  float tau;              /* SALE threshold on the relative score, 0 < tau <= 1 */
  float softmax_scale;    /* > 0, or 0 for 1/sqrt(head_dim) */
  uint32_t wait_limit_us; /* bound on every device-side wait; 0 -> 250,000 us */
  uint32_t debug_flags;   /* 0 in normal use; SPA_DEBUG_* test hooks */
  const float* tau_per_head; /* SALE: optional host array of Hq thresholds (one per q head,
                                each in (0, 1]; Hq <= SPA_MAX_TAU_HEADS), read during
                                sparse_prefill_plan; NULL -> `tau` for every head */
} spa_params;

#define SPA_MAX_TAU_HEADS 128

/* Test hook: the attention kernel's MMA warp additionally waits on a barrier
 * that nothing ever signals, so its bounded wait expires after wait_limit_us;
 * the kernel then records SPA_ERR_TIMEOUT and returns without faulting. */
#define SPA_DEBUG_STALL_ATTN 0x1u


typedef struct {
  uint32_t error_bits;       /* device error word: bit0 timeout, bit1 bad index */
  uint32_t reserved;
  int64_t query_blocks;      /* B * Hq * ceil(L / block_q) */
  int64_t candidates;        /* sum over blocks of |C_b| (keys) */
  int64_t kept_candidates;   /* sum over blocks of kept candidate keys */
  int64_t kept_pairs;        /* sum over rows of |K_i|; kept FLOPs = 4 * head_dim * kept_pairs */
  int64_t dense_pairs;       /* sum over rows of (i + 1): the causal dense count */
} spa_stats;

/* Bytes of device workspace sparse_prefill_plan/attn need for these params
 * (closed form; 0 when the params are invalid).
 *
 * Workspace layout (byte offsets; A(x) rounds x up to a multiple of 256;
 * NB = B * Hq * ceil(L / 128); blocks are ordered (b, h, qb)):
 *   [0, 256)            header: uint32 error word at 0, 5 int64 counters at 8;
 *   256                 counts: int32[NB], kept candidates of each block
 *                       (keys in ANCHOR mode, key blocks in SALE mode);
 *   A(256 + 4 * NB)     lists: int32, ascending.  The list of block (b, h, qb)
 *                       starts at element (b * Hq + h) * P(nqb) + P(qb) with
 *                       P(n) = sum_{q < n} max(0, (q + 1) * 128 - local - sink)
 *                       in ANCHOR mode (key indices) and P(n) / block_k in
 *                       SALE mode (key-block indices kb: keys [kb*block_k,
 *                       (kb+1)*block_k)); capacity |C_b| keys per block;
 *   after the lists     mode-specific scratch (opaque).
 * DENSE mode uses only the header and the counts. */
SPA_API size_t sparse_prefill_workspace_bytes(const spa_params* p);

/* Selection.  Reads q, k; writes the index lists and counts into workspace.
 * ANCHOR: anchor/pool kernel, then the pooled-score scan (tensor cores) fused
 *         with the compaction (a separate bitmask pass when step is not a
 *         power of two <= 32).
 * SALE:   K mean, int4 quantisation of Q and K, sink-local statistics fused
 *         with the int8 tensor-core block scan, compaction.
 * DENSE:  only resets the workspace header. */
SPA_API spa_status sparse_prefill_plan(const spa_params* p, const void* q, const void* k,
                               void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* Attention over sink + selected + local keys (all causal keys in DENSE
 * mode).  Reads q, k, v and the plan's selection in the workspace (with
 * Hq / Hkv even, the per-tile keep masks the plan writes in its scratch
 * beside the lists; otherwise the lists); writes o and, when lse is not
 * NULL, lse.  Records device-side errors in the workspace error word. */
SPA_API spa_status sparse_prefill_attn(const spa_params* p, const void* q, const void* k,
                               const void* v, void* workspace, size_t workspace_bytes,
                               void* o, float* lse, cudaStream_t stream);

/* Reduces the plan's counts into *out (host pointer) and synchronises the
 * stream.  Returns SPA_ERR_TIMEOUT / SPA_ERR_INVALID when the error word is
 * set, after filling *out. */
SPA_API spa_status sparse_prefill_stats(const spa_params* p, const void* workspace,
                                size_t workspace_bytes, spa_stats* out,
                                cudaStream_t stream);

/* Allocation-free selection (ANCHOR mode only).  The paper has no
 * counterpart: this entry point exists for callers that cannot give the
 * library a workspace -- plugin hosts whose enqueue step may not allocate
 * device memory, serving stacks that reserve their whole memory budget at
 * start-up, and hot paths that must not call cudaMalloc because it can
 * synchronise the device.  It computes exactly what sparse_prefill_plan
 * computes, but the scratch (header, anchor means, pooled queries, key
 * bitmask) lives in a fixed device array of SPA_STATIC_SCRATCH_BYTES inside
 * the library, which every GPU that loads the library holds until the
 * process exits.  Nothing is allocated or freed.
 *
 *   q, k        inputs as for sparse_prefill_plan (device, 16-byte aligned);
 *   counts      output, device int32[B*Hq*ceil(L/128)], blocks in (b, h, qb) order;
 *   lists       output, device int32[lists_elems]: the block lists at the
 *               offsets documented for the workspace's list region, relative
 *               to `lists` (B*Hq*P(nqb) elements are needed);
 *   error_word  optional device uint32 that receives the device error word
 *               (bit0 timeout, bit1 bad index) after the call; may be NULL.
 *
 * Returns SPA_ERR_UNSUPPORTED when the mode is not ANCHOR or when the scratch
 * these params need exceeds SPA_STATIC_SCRATCH_BYTES (about B*Hq*L*L/1024
 * bytes of bitmask plus 516 bytes per query block; 32 q heads fit up to
 * L = 32768), SPA_ERR_WORKSPACE when lists_elems is too small, and the same
 * argument errors as sparse_prefill_plan, all before any launch.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  A call that finds the device's context changed
 * since (after cudaDeviceReset) looks the address up again, so it too should
 * come before any capture.  For an empty problem (B or L zero) nothing is
 * launched and *error_word, when given, is set to zero.  All calls share the array and it keeps the last
 * call's contents (the header is cleared on every call); calls that overlap
 * on the GPU -- on different streams or from different threads -- race and
 * must be serialised by the caller. */
#define SPA_STATIC_SCRATCH_BYTES ((size_t)48 << 20)
SPA_API spa_status sparse_prefill_plan_static(const spa_params* p, const void* q, const void* k,
                                              int32_t* counts, int32_t* lists,
                                              size_t lists_elems, uint32_t* error_word,
                                              cudaStream_t stream);

/* Decode-shaped reuse of a finished plan (SpotAttention, Fig. 2 and Sec. 3:
 * a decoding query attends to a sink prefix, a recency window and a set of
 * selected blocks).  The selected part is the plan's selection for the last
 * prompt query block qb = (L - 1) / 128, so one query per (b, q head) at
 * absolute position pos (L - 1 <= pos < kv_capacity, the same for every
 * sequence) attends to
 *
 *   D_h(pos) = [0, min(sink, pos + 1)) u sel_h(qb) u [max(ls_qb, min(sink, pos + 1)), pos],
 *
 * every key up to pos in DENSE mode.  At pos = L - 1 this is the key set the
 * prefill gave its last prompt row.  p is the plan's params (seq_len = L, the
 * prompt length); the workspace is the plan's and is only read, except for
 * its error word.
 *
 *   scratch      caller-owned device buffer of sparse_decode_scratch_bytes
 *                (16-byte aligned) shared by prepare and attn: the union of
 *                each kv head's q heads' selections and the split partials;
 *   kv_capacity  rows per (b, kv head) of the K/V cache, L <= kv_capacity <= 2^24;
 *   q            bf16 [B, Hq, 128], the decoding queries;
 *   k_cache, v_cache  bf16 [B, Hkv, kv_capacity, 128]; rows 0..pos must hold
 *                the keys/values of positions 0..pos (the prompt's at 0..L-1);
 *   o            bf16 [B, Hq, 128]; lse: optional fp32 [B, Hq] (natural log).
 *
 * sparse_decode_prepare runs once per plan (it merges the selections of the
 * q heads of each kv head into one list with per-head bits); every
 * sparse_decode_attn call after it, at any pos, reuses that list until the
 * next plan or prepare on the same buffers.  Argument errors are returned
 * before any launch; a list entry outside its block's candidates sets the
 * bad-index bit of the workspace error word (reported by
 * sparse_prefill_stats). */
SPA_API size_t sparse_decode_scratch_bytes(const spa_params* p, int32_t kv_capacity);
SPA_API spa_status sparse_decode_prepare(const spa_params* p, int32_t kv_capacity,
                                         void* workspace, size_t workspace_bytes, void* scratch,
                                         size_t scratch_bytes, cudaStream_t stream);
SPA_API spa_status sparse_decode_attn(const spa_params* p, const void* q, const void* k_cache,
                                      const void* v_cache, int32_t kv_capacity, int32_t pos,
                                      void* workspace, size_t workspace_bytes, void* scratch,
                                      size_t scratch_bytes, void* o, float* lse,
                                      cudaStream_t stream);

/* FP8 attention (SALE's Computation Pass on quantised operands,
 * "SageAttention-style": the review of SALE, Summary), on the tcgen05
 * kind::f8f6f4 tensor cores.  Two calls:
 *
 * sparse_fp8_quantize writes E4M3 codes (OCP "fn": bias 7, 3 mantissa bits,
 * largest finite 448; round to nearest even, saturating) of q, k, v:
 *   q8       uint8 [B, Hq, L, 128], one scale per (b, q head, 128-row block);
 *   k8       uint8 [B, Hkv, L, 128] of K minus its per-(b, kv head) sequence
 *            mean (fp64 sum / L rounded once to fp32; a constant shift of each
 *            row's scores), one scale per (b, kv head);
 *   v8       uint8 [B, Hkv, L, 128], one scale per (b, kv head, channel);
 *   scales   fp32 [sparse_fp8_scales_floats(p)] = q scales [B*Hq*nqb], k scales
 *            [B*Hkv], v scales [B*Hkv*128], K means [B*Hkv*128], in that order;
 * scale = absmax / 448 in IEEE fp32 (1 for an all-zero group); code =
 * E4M3(x / scale) with an IEEE fp32 division.  scratch: device buffer of
 * sparse_fp8_scratch_bytes(p), 16-byte aligned, contents not kept.
 *
 * sparse_prefill_attn_fp8 runs the attention of sparse_prefill_attn over the
 * plan in the workspace (mode, sink, local as planned) with the dequantised
 * operands: P is rounded to E4M3 before the PV product (relative error
 * <= 2^-4 each), O is bf16 [B, Hq, L, 128], and lse (optional, fp32
 * [B, Hq, L], natural log) is that of the scores against the unsmoothed
 * dequantised keys (the mean shift is added back).
 *
 * Pointers are device pointers, 16-byte aligned (scales and lse 4-byte).
 * Argument errors are returned before any launch; device-side errors set the
 * workspace error word as for sparse_prefill_attn. */
SPA_API size_t sparse_fp8_scales_floats(const spa_params* p);
SPA_API size_t sparse_fp8_scratch_bytes(const spa_params* p);
SPA_API spa_status sparse_fp8_quantize(const spa_params* p, const void* q, const void* k,
                                       const void* v, void* q8, void* k8, void* v8,
                                       float* scales, void* scratch, size_t scratch_bytes,
                                       cudaStream_t stream);
SPA_API spa_status sparse_prefill_attn_fp8(const spa_params* p, const void* q8, const void* k8,
                                           const void* v8, const float* scales, void* workspace,
                                           size_t workspace_bytes, void* o, float* lse,
                                           cudaStream_t stream);

/* Attention mass per key from the prefill rows, reusing the prefill LSE
 * (KVpop, Sec. 3: the future attention mass of a token, from a transposed
 * attention pass over the sparse kept sets with the sparse LSE normalisers,
 * aggregated over the query heads that share a kv head):
 *
 *   mass[b, g, j] = sum over q heads h of kv head g, and over rows i whose
 *                   kept set (as planned in the workspace) holds j and with
 *                   i - j >= window, of exp(s_ij - lse[b, h, i]),
 *
 * s_ij the scaled score of q_i and k_j.  q, k as for sparse_prefill_plan;
 * lse fp32 [B, Hq, L] (natural log; normally sparse_prefill_attn's output
 * for the same plan); mass fp32 [B, Hkv, L], overwritten.  window >= 0, and
 * window <= local - block_q outside DENSE mode (every selected key then lies
 * at least that far behind every row of its block).  Errors as for
 * sparse_prefill_attn. */
SPA_API spa_status sparse_key_mass(const spa_params* p, const void* q, const void* k,
                                   const float* lse, int32_t window, void* workspace,
                                   size_t workspace_bytes, float* mass, cudaStream_t stream);

/* Static string for a status code. */
SPA_API const char* sparse_prefill_status_string(spa_status s);

#ifdef __cplusplus
}
#endif

#endif /* SPA_H_ */
