// kernels.h -- launch parameters shared between the C-ABI layer (api.cu) and
// the kernel translation units.  Internal; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace attn {

// Fixed geometry of this build.
constexpr int kPrefillBlockM = 128;   // query rows per tcgen05 tile
constexpr int kPrefillBlockN = 128;   // keys per S = Q K^T MMA tile
constexpr int kSkipTile = 32;         // keys per skip-softmax unit
constexpr int kDecodeSplits = 32;     // dense decode schedule: KV splits
constexpr int kDecodeSplitTile = 128; // dense decode schedule: keys per tile
constexpr int kPageSize = 16;
constexpr int kSmallSeqMaxKv = 16;
constexpr int kMaxGroup = 16;         // largest h_q / h_kv supported by decode

struct SmallSeqParams {
  const uint16_t *q, *k, *v;
  const int32_t *cu;
  uint16_t *out, *weights;             // forward outputs (weights may be null)
  const uint16_t *dout, *weights_in;   // backward inputs: dO and the forward's weights
  uint16_t *dq, *dk, *dv;              // backward outputs
  int batch, total_kv, h, d, max_s_kv;
  float scale_log2, scale;
  unsigned int *err;
};

struct BwdParams {
  const int32_t *cu_q, *cu_k;
  const uint16_t *out, *dout;   // [total_q, h_q, d] the forward's output and its gradient
  const float *lse;             // [total_q, h_q] the forward's log-sum-exp (natural log)
  float *delta;                 // [total_q, h_q] workspace: <dO, O> per row
  uint16_t *dq;                 // [total_q, h_q, d]
  uint16_t *dk, *dv;            // [total_k, h_kv, d]
  int batch, total_q, total_k, max_q, max_k, h_q, h_kv, group, d, causal;
  int qb_max, kt_max;           // ceil(max_q / 128), ceil(max_k / 128)
  float scale, scale_log2;
  unsigned int *err;
};

struct DecodeParams {
  const uint16_t *q;            // [B, h_q, d]
  const int32_t *block_table;   // [B, max_pages]
  const int32_t *seq_lens;      // [B]
  uint16_t *out;                // [B, h_q, d]
  float *lse;                   // [B, h_q] or null
  float *ws_o;                  // [B, h_q, splits, d]   (split schedules)
  float *ws_ml;                 // [B, h_q, splits, 2]   (split schedules)
  float *ws_s;                  // [B, h_kv, max_pages * 16, G] scores (two-pass skip)
  float *ws_tmax;               // [B, h_kv, kt_max, G] 32-key tile maxima (two-pass skip)
  float *ws_smax;               // [B, h_kv, splits, G] split maxima (two-pass skip)
  // one-pass skip schedule: [B, h_kv, splits, G] published split maxima (high
  // word 1 once written, low word the fp32 bits; zeroed before the launch),
  // the launch's work-ticket counter (zeroed before the launch), and the most
  // keys a split holds (its scores stay in shared memory)
  unsigned long long *ws_pub;
  unsigned int *ws_ticket;
  int split_keys;
  uint32_t *skip_mask;          // or null
  unsigned long long *skip_counts;  // or null
  int batch, h_q, h_kv, group, d, num_pages, max_pages, kt_max;
  int s_stride;                 // key slots per (sequence, kv-head) in ws_s: max_pages * 16 rounded up to 64
  float scale_log2;             // scale * log2(e)
  float thr_log2;               // log2(threshold); -inf when skipping is off
  int sequential;               // skip mode: 1 = one split walking 32-key tiles, 2 = two passes,
                                // 3 = one pass over the splits (each waits for the earlier splits' maxima)
  // NVFP4 quantise-dequantise of P and / or V (skip schedules only): which
  // operands, their 448 / amax, their ratio tables g / (1 + j / 8), j = 0..7
  // (g = 2688 / amax, fp32), and the output factor 1 / g over the quantised
  // operands
  int p_qdq, v_qdq;
  float p_k, v_k;
  float p_tab[8], v_tab[8];
  float qdq_out;
  unsigned int *err;
};

struct PrefillParams {
  const int32_t *cu_q, *cu_k;
  uint16_t *out;
  float *lse;
  uint32_t *skip_mask;
  unsigned long long *skip_counts;
  int batch, total_q, total_k, max_q, max_k, h_q, h_kv, group, d, causal;
  int qb_max, kt_max;           // ceil(max_q / 128), ceil(max_k / 32)
  float scale_log2, thr_log2;
  unsigned int *err;
  int work_slot;                // work-claim slot of this launch (set by launch_prefill)
  uint32_t work_tag;            // nonzero tag of this launch in its slot (set by launch_prefill)
  // item order: 0 = query blocks outermost (heaviest causal block first, for
  // s_q = s_k); 1 = sequences outermost (all items that read one sequence's
  // K/V run together, for prefixes longer than the queries)
  int seq_major;
  // paged K/V (chunked prefill): keys and values of sequence b live in the
  // pages block_table[b, :] of a [num_pages, 16, h_kv, d] cache, s_k =
  // seq_lens_k[b]; cu_k / total_k are unused then
  int paged, num_pages, max_pages;
  const int32_t *block_table, *seq_lens_k;
};

cudaError_t launch_smallseq(const SmallSeqParams &p, cudaStream_t stream);
cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                            const CUtensorMap &vmap, const CUtensorMap &dmap, cudaStream_t stream);
cudaError_t launch_smallseq_bwd(const SmallSeqParams &p, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream);
// Shared memory of the one-pass skip schedule for splits of up to `split_keys`
// keys and groups of `group` heads (0 when it does not fit one CTA).
size_t decode_one_pass_smem(int d, int group, int split_keys);
cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &qmap,
                           const CUtensorMap &kmap, const CUtensorMap &vmap, const CUtensorMap &omap,
                           cudaStream_t stream);

}  // namespace attn
