/*
 * attn.h -- C ABI of the B200 (sm_100a) fused attention-forward library.
 *
 * Three operations, all computing masked softmax(Q K^T * scale) V with an
 * online (flash-attention style) softmax:
 *
 *   attn_varlen_fwd     packed variable-length GQA prefill, causal or not
 *                       (NVIDIA/Model-Optimizer PR 1034, "Add Triton unified
 *                       attention kernel with HuggingFace integration":
 *                       variable-length batching, GQA, causal/non-causal),
 *                       and attn_varlen_bwd, its gradients.
 *   attn_paged_decode   one query token per sequence against a paged KV cache
 *                       (NVIDIA/Model-Optimizer PR 1941, "Add split-k decode
 *                       kernel for skip softmax": a 32-split schedule of
 *                       128-token tiles when skip-softmax is off, one
 *                       sequential split of 32-token tiles when it is on).
 *   attn_smallseq_fwd   s_q = 1, s_kv <= 16 cross attention over a huge batch,
 *                       also returning the attention weights
 *                       (ROCm/TransformerEngine PR 461, "Integrate CK varlen
 *                       cross attention for small-seq (s_q=1, s_kv<=16)"),
 *                       and attn_smallseq_bwd, its gradients from those weights.
 *
 * Skip-softmax (NVIDIA/TensorRT-LLM PR 9821, "Skip Softmax Attention"):
 * keys are visited in 32-key tiles in increasing order; a tile is skipped for
 * a group of query rows when, for every row of the group,
 * exp(tile_max - running_max) < skip_threshold.  A skipped tile contributes
 * nothing to the output or its normaliser.  The threshold is a runtime float
 * in [0, 1]; 0 disables skipping.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE memory owned by the caller; the library
 *    allocates nothing and keeps no pointer after the call returns.
 *  - bf16 tensors are passed as attn_bf16 (raw 16-bit patterns), row-major,
 *    contiguous, base pointers 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work on it and returns; nothing synchronises.
 *  - scale: the softmax scale applied to Q.K; must be finite and > 0.  Pass
 *    1/sqrt(d) for the usual scaling.
 *  - Query head hq reads KV head hq / (h_q / h_kv) (consecutive grouping).
 *  - Causal masking is bottom-right aligned: query row i of a sequence with
 *    s_q queries and s_k keys sees keys j <= i + s_k - s_q.
 *  - A query row with no visible key gets output 0 and LSE -inf.
 *  - LSE outputs are float32 natural-log log-sum-exp of the scaled scores
 *    over the kept keys.
 *  - Host-checkable argument errors return a negative ATTN_E_* code and
 *    launch nothing.  Errors that depend on device data (bad cu_seqlens,
 *    block-table entries, over-long rows) set a bit in a per-device error
 *    word (ATTN_DEVERR_*) and the affected unit writes zeros; read and clear
 *    it with attn_get_last_device_error().
 *  - All entry points are thread-safe; concurrent calls on different streams
 *    share only the device error word.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

typedef uint16_t attn_bf16;
typedef void *attn_stream_t; /* a cudaStream_t */

enum attn_status {
  ATTN_OK = 0,
  ATTN_E_NULL = -1,        /* a required pointer is NULL                         */
  ATTN_E_ALIGN = -2,       /* a tensor pointer is not 16-byte aligned            */
  ATTN_E_HEADS = -3,       /* h_q or h_kv < 1, h_q % h_kv != 0, or group > 16    */
  ATTN_E_HEAD_DIM = -4,    /* head dim d not 64 or 128                           */
  ATTN_E_THRESHOLD = -5,   /* skip threshold NaN or outside [0, 1]               */
  ATTN_E_PAGE_SIZE = -6,   /* page_size other than 16                            */
  ATTN_E_SMALLSEQ = -7,    /* max_s_kv outside [1, 16]                           */
  ATTN_E_SHAPE = -8,       /* negative size, or max length <= 0 with work to do  */
  ATTN_E_WORKSPACE = -9,   /* workspace NULL or smaller than the query says      */
  ATTN_E_SCALE = -10,      /* scale not finite or not > 0                        */
  ATTN_E_CUDA = -11,       /* a CUDA call failed (launch, tensor-map encode ...) */
  ATTN_E_DEVICE = -12,     /* current device is not compute capability 10.x      */
  ATTN_E_TOO_LARGE = -13,  /* a size exceeds a documented implementation limit   */
  ATTN_E_QDQ = -14         /* unknown QDQ format, or amax outside [2^-64, 2^64]  */
};

/* Quantise-dequantise formats of attn_paged_decode_qdq. */
enum attn_qdq_format {
  ATTN_QDQ_NONE = 0,       /* the operand stays as it is                         */
  ATTN_QDQ_NVFP4 = 1       /* NVFP4: E2M1 values, E4M3 scales per 16, fp32 amax  */
};

/* Bits of the per-device error word. */
enum attn_device_error {
  ATTN_DEVERR_CU_SEQLENS = 1u << 0,  /* cu_seqlens not monotone, or beyond total / max     */
  ATTN_DEVERR_SEQ_LEN = 1u << 1,     /* decode seq_len < 0 or > max_pages_per_seq*page    */
  ATTN_DEVERR_BLOCK_TABLE = 1u << 2, /* block-table entry outside [0, num_pages)          */
  ATTN_DEVERR_SMALLSEQ_LEN = 1u << 3,/* small-seq row with s_kv > max_s_kv                */
  ATTN_DEVERR_TIMEOUT = 1u << 4,     /* a pipeline wait gave up (kernel returned early)   */
  ATTN_DEVERR_BUSY = 1u << 5         /* a prefill work-claim slot stayed held by another
                                        launch past the wait limit (rows not written)    */
};

/* Compile-time tile geometry of this build (reported for the tests). */
typedef struct attn_config {
  int prefill_block_m;      /* query rows per prefill tile (tcgen05 M)            */
  int prefill_block_n;      /* keys per prefill MMA tile                          */
  int skip_tile;            /* keys per skip-softmax unit (prefill and decode)    */
  int decode_splits;        /* KV splits of the dense decode schedule             */
  int decode_split_tile;    /* keys per tile of the dense split schedule          */
  int decode_page_size;     /* the only supported page size                       */
  int smallseq_max_s_kv;    /* largest supported small-seq key count              */
} attn_config;

/* Fills *cfg; returns ATTN_OK (ATTN_E_NULL if cfg is NULL). */
ATTN_API int attn_get_config(attn_config *cfg);

/* Human-readable name of a status code (static string). */
ATTN_API const char *attn_status_string(int status);

/*
 * attn_varlen_fwd -- packed varlen GQA attention forward (prefill).
 *
 *   q            [total_q, h_q, d]  bf16
 *   k, v         [total_k, h_kv, d] bf16
 *   cu_seqlens_q [batch + 1] int32, exclusive prefix sums, cu[0] = 0,
 *                cu[batch] <= total_q   (same for cu_seqlens_k / total_k)
 *   max_q, max_k upper bounds of the per-sequence lengths (size the grid);
 *                a sequence longer than them sets ATTN_DEVERR_CU_SEQLENS
 *   d            64 or 128
 *   out          [total_q, h_q, d] bf16 (written for every row of every
 *                sequence; rows outside [cu[0], cu[batch]) are untouched)
 *   lse          [total_q, h_q] float32, may be NULL
 *
 * Work balance: the kernel's CTAs claim work items from a counter the library
 * keeps in device memory, one of 64 per device taken in turn by successive
 * launches (attn_varlen_fwd, attn_varlen_fwd_ex and attn_paged_prefill
 * alike).  Each launch tags its counter and frees it with its last claim; a
 * launch that meets a counter still held by another waits until it is freed
 * (at most about one second), so any number of these calls may run
 * concurrently on one device.  A wait that runs out sets ATTN_DEVERR_BUSY
 * and the waiting part of the launch writes nothing.  Two concurrent replays
 * of one captured CUDA graph share its launches' tags and must not overlap
 * (they would also write the same outputs).
 *
 * Returns ATTN_OK or an ATTN_E_* code (nothing launched on error).
 */
ATTN_API int attn_varlen_fwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                    int batch, int total_q, int total_k, int max_q, int max_k,
                    int h_q, int h_kv, int d, int causal, float scale,
                    attn_bf16 *out, float *lse, attn_stream_t stream);

/*
 * attn_varlen_fwd_ex -- attn_varlen_fwd with the skip-softmax tile rule.
 *
 * Units: (sequence b, q-head, q-block of prefill_block_m rows) x (key tile of
 * skip_tile keys).  The rows a unit serves are the query rows of the block
 * that belong to sequence b.  A unit is visited when at least one of its
 * (row, key) pairs is unmasked.
 *
 *   skip_threshold  in [0, 1]; 0 gives exactly attn_varlen_fwd's result
 *   skip_mask       NULL, or a bit array of
 *                   batch * ceil(max_q / block_m) * h_q * ceil(max_k / skip_tile)
 *                   bits (uint32 words, bit i of word w = unit 32w + i), unit
 *                   index ((b * QB + r) * h_q + hq) * KT + t with
 *                   QB = ceil(max_q / block_m), KT = ceil(max_k / skip_tile).
 *                   Cleared by the call; a set bit marks a skipped unit.
 *   skip_counts     NULL, or 2 uint64: {visited units, skipped units};
 *                   cleared by the call.
 */
ATTN_API int attn_varlen_fwd_ex(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int total_q, int total_k, int max_q, int max_k,
                       int h_q, int h_kv, int d, int causal, float scale,
                       float skip_threshold, uint32_t *skip_mask,
                       unsigned long long *skip_counts,
                       attn_bf16 *out, float *lse, attn_stream_t stream);

/*
 * attn_paged_prefill -- varlen GQA attention forward whose keys and values
 * live in a paged cache: chunked prefill, or several query tokens per
 * sequence against the cache (NVIDIA/Model-Optimizer PR 1941, "Add split-k
 * decode kernel for skip softmax", What does this PR do?, fifth bullet: the
 * dedicated decode kernel takes one-token decode only, and prefill and
 * multi-token decode over the paged cache stay on the general flash-attention
 * kernel).  Sequence b has
 * s_q = cu_seqlens_q[b+1] - cu_seqlens_q[b] query tokens, which are the last
 * s_q positions of its s_k = seq_lens_k[b] cached tokens when causal
 * (bottom-right alignment: query row i sees keys j <= i + s_k - s_q).
 *
 *   q              [total_q, h_q, d] bf16, packed like attn_varlen_fwd's
 *   k_cache,
 *   v_cache        [num_pages, page_size, h_kv, d] bf16; token t of sequence
 *                  b lives in page block_table[b, t / page_size], slot
 *                  t % page_size (the attn_paged_decode layout)
 *   block_table    [batch, max_pages_per_seq] int32; entries beyond a
 *                  sequence's last page are never read
 *   cu_seqlens_q   [batch + 1] int32 prefix sums over total_q
 *   seq_lens_k     [batch] int32, 0 <= seq_lens_k[b] <= min(max_k,
 *                  max_pages_per_seq * page_size)
 *   page_size      16
 *   max_q, max_k   bounds of s_q and s_k (size the grid and the skip mask)
 *   skip_threshold, skip_mask, skip_counts
 *                  as attn_varlen_fwd_ex (same units and bit layout, with
 *                  KT = ceil(max_k / skip_tile))
 *   out            [total_q, h_q, d] bf16;  lse [total_q, h_q] float32 or NULL
 *
 * Cache slots past a sequence's end in its last page may hold anything (they
 * are neither attended to nor multiplied into the output).  A block-table
 * entry outside [0, num_pages) sets ATTN_DEVERR_BLOCK_TABLE and that page is
 * read as zeros; a bad cu_seqlens_q or seq_lens_k entry sets
 * ATTN_DEVERR_CU_SEQLENS and the sequence is not written.  Shares the
 * work-claim counters of attn_varlen_fwd (see there).
 */
ATTN_API int attn_paged_prefill(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                       const int32_t *block_table, const int32_t *cu_seqlens_q,
                       const int32_t *seq_lens_k, int batch, int total_q, int max_q, int max_k,
                       int num_pages, int max_pages_per_seq, int page_size,
                       int h_q, int h_kv, int d, int causal, float scale,
                       float skip_threshold, uint32_t *skip_mask,
                       unsigned long long *skip_counts,
                       attn_bf16 *out, float *lse, attn_stream_t stream);

/*
 * attn_varlen_bwd -- gradients of attn_varlen_fwd (skip threshold 0) with
 * respect to q, k and v, for training through autograd (NVIDIA/Model-Optimizer
 * PR 1034, "Add Triton unified attention kernel with HuggingFace
 * integration", description).  With P = exp(scale * Q K^T - lse) over the
 * allowed keys (the same masks as the forward), Delta_i = <dO_i, O_i>,
 * dP = dO V^T and dS = P * (dP - Delta):
 *   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
 * dK and dV summed over the q-heads of each kv-head's group.
 *
 *   q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_q,
 *   max_k, h_q, h_kv, d, causal, scale   as passed to attn_varlen_fwd
 *   out            [total_q, h_q, d] bf16, the forward's output
 *   dout           [total_q, h_q, d] bf16, the loss gradient w.r.t. out
 *   lse            [total_q, h_q] float32, the forward's log-sum-exp (natural
 *                  log, -inf for rows with no key)
 *   dq             [total_q, h_q, d] bf16 output
 *   dk, dv         [total_k, h_kv, d] bf16 outputs; every key of a valid
 *                  sequence is written (zero when no query sees it)
 *   workspace      device buffer of >= attn_varlen_bwd_workspace_size(total_q,
 *                  h_q) bytes, 16-byte aligned (Delta per row); required
 *                  when batch > 0
 * A sequence with an invalid cu_seqlens range sets ATTN_DEVERR_CU_SEQLENS and
 * none of its rows are written.  The result is deterministic (no atomics).
 */
ATTN_API size_t attn_varlen_bwd_workspace_size(int total_q, int h_q);
ATTN_API int attn_varlen_bwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                             const attn_bf16 *out, const attn_bf16 *dout, const float *lse,
                             const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k, int batch,
                             int total_q, int total_k, int max_q, int max_k, int h_q, int h_kv, int d,
                             int causal, float scale, attn_bf16 *dq, attn_bf16 *dk, attn_bf16 *dv,
                             void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_paged_decode_workspace_size -- bytes of workspace attn_paged_decode
 * needs for this shape (a pure host query; 0 is never returned for
 * batch * h_q > 0).  The dense schedule keeps, per (sequence, q-head, split),
 * the split's running max, running sum and unnormalised output in float32.
 * The caller asks for the size first and passes a buffer of at least that
 * many bytes, the shape- and workspace-query convention of
 * ROCm/TransformerEngine PR 461 ("Integrate CK varlen cross attention for
 * small-seq (s_q=1, s_kv<=16)", description bullets: the forward and
 * backward each get a workspace-size query that the caller runs before the
 * launch).  Sizes: 32 * batch * h_q * (4 d + 8) bytes, each of its two parts
 * (outputs, then max and sum) rounded up to 256 bytes.
 */
ATTN_API size_t attn_paged_decode_workspace_size(int batch, int h_q, int d);

/*
 * attn_paged_decode_workspace_size_ex -- the same query (same convention,
 * ROCm/TransformerEngine PR 461, description bullets) for either schedule:
 * skip_threshold == 0 gives attn_paged_decode_workspace_size(batch, h_q, d);
 * skip_threshold > 0 gives the two-pass skip schedule's need: the split
 * partials plus, in float32, the scores of every (query head, key slot up to
 * max_pages_per_seq * 16, rounded up to 64), the maxima of every 32-key tile
 * and of every split (about batch * h_q * max_pages_per_seq * 64 bytes).  The
 * one-pass form of that schedule uses the same workspace (the partials, and
 * at the start of the scores area a work counter and the published split
 * maxima, zeroed by the call in its stream).
 */
ATTN_API size_t attn_paged_decode_workspace_size_ex(int batch, int h_q, int d, int max_pages_per_seq,
                                                    float skip_threshold);

/*
 * attn_paged_decode -- one query token per sequence against a paged cache.
 *
 *   q              [batch, h_q, d] bf16
 *   k_cache,
 *   v_cache        [num_pages, page_size, h_kv, d] bf16; token t of sequence
 *                  b lives in page block_table[b, t / page_size], slot
 *                  t % page_size
 *   block_table    [batch, max_pages_per_seq] int32; entries beyond a
 *                  sequence's last page are never read
 *   seq_lens       [batch] int32, 0 <= seq_lens[b] <= max_pages_per_seq*page_size
 *   page_size      16
 *   skip_threshold 0: dense split-KV schedule (32 splits of 128-key tiles per
 *                  (sequence, kv-head)) followed by a log-sum-exp combine;
 *                  > 0 (and <= 1): skip-softmax over 32-key tiles visited in
 *                  order; a tile is skipped when all h_q / h_kv query heads
 *                  of the group vote skip against the running max.  With a
 *                  workspace this runs over the split schedule: a skipped
 *                  tile never raises the running max, so the max entering a
 *                  tile is the max of all earlier tiles, and a split that
 *                  knows the earlier splits' maxima takes the sequential
 *                  walk's decisions.  When a split's scores fit one CTA's
 *                  shared memory (keys per split * h_q / h_kv * 4 bytes, with
 *                  the rest of the CTA's state, within 56 KB, so that four
 *                  CTAs share an SM) it is one pass: each split's CTA computes its scores, publishes its
 *                  maximum, waits for the earlier splits' and copies the
 *                  kept tiles' V; otherwise two passes (scores and tile
 *                  maxima to the workspace, then the kept tiles' P V).  With
 *                  workspace NULL it runs as one sequential split per
 *                  (sequence, kv-head).  All give the same decisions.
 *   out            [batch, h_q, d] bf16
 *   lse            [batch, h_q] float32, may be NULL
 *   workspace      device buffer of >= attn_paged_decode_workspace_size_ex(
 *                  batch, h_q, d, max_pages_per_seq, skip_threshold) bytes,
 *                  16-byte aligned; required when skip_threshold is 0, NULL
 *                  (sequential skip schedule) or such a buffer otherwise
 */
ATTN_API int attn_paged_decode(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                      const int32_t *block_table, const int32_t *seq_lens,
                      int batch, int num_pages, int max_pages_per_seq, int page_size,
                      int h_q, int h_kv, int d, float skip_threshold, float scale,
                      attn_bf16 *out, float *lse,
                      void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_paged_decode_ex -- attn_paged_decode plus skip-softmax reporting.
 *
 *   skip_mask    NULL, or a bit array of batch * h_kv * ceil(max_pages_per_seq
 *                * page_size / skip_tile) bits, unit index (b * h_kv + hk) * KT + t;
 *                cleared by the call.
 *   skip_counts  NULL, or 2 uint64 {visited tiles, skipped tiles}; cleared.
 */
ATTN_API int attn_paged_decode_ex(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                         const int32_t *block_table, const int32_t *seq_lens,
                         int batch, int num_pages, int max_pages_per_seq, int page_size,
                         int h_q, int h_kv, int d, float skip_threshold, float scale,
                         uint32_t *skip_mask, unsigned long long *skip_counts,
                         attn_bf16 *out, float *lse,
                         void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_paged_decode_qdq -- attn_paged_decode_ex with NVFP4 quantise-dequantise
 * (QDQ) of the probabilities P and / or the values V before their product
 * (NVIDIA/Model-Optimizer PR 1941, "Add split-k decode kernel for skip
 * softmax", What does this PR do?, third bullet: skip-softmax together with
 * NVFP4 P/V QDQ; Usage: p_qdq="nvfp4", p_qdq_amax, v_qdq="nvfp4",
 * v_qdq_amax).  The page prints no recipe; this library's reading:
 *
 *   - blocks of 16 along the key axis (the contraction axis of P V): P per
 *     query head over 16 consecutive keys, V per channel over 16 consecutive
 *     keys (one page) of each kv-head;
 *   - per block, with k = 448 / amax and g = 2688 / amax (fp32): s =
 *     E4M3(max|x| * k), q = E2M1(x * (g / s)) (both round to nearest even and
 *     saturate), dequantised value q * s / g; the code-deciding products and
 *     the quotient g / s are fp32, correctly rounded;
 *   - p = exp(score - M_t), M_t the running max of the 32-key walk after the
 *     key's tile; the softmax normaliser sums the unquantised p, so the LSE
 *     output is that of attn_paged_decode;
 *   - with either operand quantised the decode always runs a 32-key skip
 *     schedule (threshold 0 skips nothing): two passes over the splits with a
 *     workspace of attn_paged_decode_qdq_workspace_size() bytes, or one
 *     sequential split per (sequence, kv-head) with workspace NULL.
 *
 *   p_qdq, v_qdq        ATTN_QDQ_NONE or ATTN_QDQ_NVFP4
 *   p_qdq_amax,
 *   v_qdq_amax          the operand's calibrated absolute maximum, finite, in
 *                       [2^-64, 2^64] when its format is NVFP4 (ignored
 *                       otherwise); values above it saturate.  Probabilities
 *                       never exceed 1, so 1 is the natural P amax.
 *   other arguments     as attn_paged_decode_ex.  With both formats NONE
 *                       the call is attn_paged_decode_ex.
 * Errors as attn_paged_decode_ex, plus ATTN_E_QDQ.
 */
ATTN_API size_t attn_paged_decode_qdq_workspace_size(int batch, int h_q, int d, int max_pages_per_seq);
ATTN_API int attn_paged_decode_qdq(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                                   const int32_t *block_table, const int32_t *seq_lens, int batch,
                                   int num_pages, int max_pages_per_seq, int page_size, int h_q, int h_kv,
                                   int d, float skip_threshold, float scale, int p_qdq, float p_qdq_amax,
                                   int v_qdq, float v_qdq_amax, uint32_t *skip_mask,
                                   unsigned long long *skip_counts, attn_bf16 *out, float *lse,
                                   void *workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_paged_decode_static -- attn_paged_decode for callers that cannot
 * allocate device memory.  (The source pages have no counterpart; this entry
 * point exists only for such callers.)
 *
 * Some callers cannot hand the library a workspace: a serving runtime whose
 * memory pool already owns the whole GPU and treats any further cudaMalloc
 * as an error, or a plug-in interface that has no workspace argument and
 * runs where a cudaMalloc (which may synchronise the device) is not
 * allowed.  This variant takes the same arguments as attn_paged_decode minus
 * the workspace and keeps the split-KV partials in a scratch array that the
 * library itself holds in device memory:
 *
 *   - scratch limit: ATTN_STATIC_WORKSPACE_BYTES (48 MiB).  A dense-mode
 *     shape whose attn_paged_decode_workspace_size(batch, h_q, d) exceeds it
 *     returns ATTN_E_TOO_LARGE and launches nothing: the shape fits when
 *     32 * batch * h_q * (4 d + 8) bytes, with the two parts (outputs, then
 *     max and sum) each rounded up to 256, is at most 48 MiB, i.e.
 *     batch * h_q <= 3024 at d = 128 and <= 5957 at d = 64.  In skip mode the split
 *     schedule (one or two passes) runs when its workspace fits the array,
 *     the sequential one (no workspace) otherwise.
 *   - every GPU that loads the library reserves those 48 MiB until the
 *     process exits.
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) for that device; make that first call before
 *     any stream capture begins.
 *   - all calls share the one array and it keeps whatever the last call left
 *     in it (nothing there has to start at zero: every split writes its own
 *     partial before the combine reads it).  Calls that can overlap on the
 *     GPU -- on different streams without ordering between them -- race on
 *     it and give wrong results; order them on one stream or use
 *     attn_paged_decode with a workspace per stream.
 *   - no cudaMalloc, cudaFree or other allocating routine is called.
 *   - argument errors are checked, and reported with the same codes, as by
 *     attn_paged_decode_ex; ATTN_E_TOO_LARGE comes after those checks.
 */
#define ATTN_STATIC_WORKSPACE_BYTES ((size_t)48 << 20)
ATTN_API int attn_paged_decode_static(const attn_bf16 *q, const attn_bf16 *k_cache,
                                      const attn_bf16 *v_cache, const int32_t *block_table,
                                      const int32_t *seq_lens, int batch, int num_pages,
                                      int max_pages_per_seq, int page_size, int h_q, int h_kv,
                                      int d, float skip_threshold, float scale, attn_bf16 *out,
                                      float *lse, attn_stream_t stream);

/*
 * attn_smallseq_fwd -- one query per sequence, at most 16 keys each.
 *
 *   q              [batch, h, d] bf16 (batch = number of query tokens)
 *   k, v           [total_kv, h, d] bf16
 *   cu_seqlens_kv  [batch + 1] int32 prefix sums of the per-sequence key counts
 *   max_s_kv       runtime upper bound of the key counts, 1..16; it is the last
 *                  dimension of `weights`.  A row with more keys sets
 *                  ATTN_DEVERR_SMALLSEQ_LEN and writes zeros.
 *   out            [batch, h, d] bf16
 *   weights        NULL, or [batch, h, 1, max_s_kv] bf16: the softmax
 *                  probabilities, zero beyond the row's own key count
 * Non-causal; h_q = h_kv = h.
 */
ATTN_API int attn_smallseq_fwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                      const int32_t *cu_seqlens_kv, int batch, int total_kv, int h, int d,
                      int max_s_kv, float scale, attn_bf16 *out, attn_bf16 *weights,
                      attn_stream_t stream);

/*
 * attn_smallseq_bwd -- gradients of attn_smallseq_fwd with respect to q, k
 * and v, computed from the attention weights the forward returned
 * (ROCm/TransformerEngine PR 461, description bullets: the backward's steps
 * are grad_V, grad_attn, softmax backward and grad_Q / grad_K, and it reads
 * the weights the forward wrote instead of recomputing them).  For token b,
 * head hh, keys j of the token and P_j = weights[b, hh, 0, j]:
 *   dV_j = P_j dO,  dP_j = <dO, v_j>,  dS_j = P_j (dP_j - sum_i P_i dP_i),
 *   dQ = scale sum_j dS_j k_j,  dK_j = scale dS_j q.
 *
 *   q, k, v, cu_seqlens_kv, batch, total_kv, h, d, max_s_kv, scale
 *                  as passed to attn_smallseq_fwd
 *   dout           [batch, h, d] bf16: gradient of the loss w.r.t. `out`
 *   weights        [batch, h, 1, max_s_kv] bf16, as attn_smallseq_fwd wrote it
 *                  (required)
 *   dq             [batch, h, d] bf16 output
 *   dk, dv         [total_kv, h, d] bf16 outputs.  Every key inside a valid
 *                  row's range is written once; keys outside every valid
 *                  row's range (none when cu_seqlens_kv runs from 0 to
 *                  total_kv) are left untouched.
 * A row whose key range is invalid sets ATTN_DEVERR_CU_SEQLENS, a row with
 * more than max_s_kv keys ATTN_DEVERR_SMALLSEQ_LEN; such a row's dq is zero
 * and its keys' dk, dv are not written.  Empty rows give dq = 0.
 */
ATTN_API int attn_smallseq_bwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                               const attn_bf16 *dout, const attn_bf16 *weights,
                               const int32_t *cu_seqlens_kv, int batch, int total_kv, int h, int d,
                               int max_s_kv, float scale, attn_bf16 *dq, attn_bf16 *dk,
                               attn_bf16 *dv, attn_stream_t stream);

/*
 * attn_get_last_device_error -- synchronises `stream`, then returns and
 * clears the current device's error word (a mask of ATTN_DEVERR_* bits), or
 * a negative ATTN_E_CUDA if the synchronisation itself failed.
 */
ATTN_API int attn_get_last_device_error(attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
