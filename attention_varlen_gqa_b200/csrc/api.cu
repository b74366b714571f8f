// api.cu -- the C ABI declared in include/attn.h: argument validation,
// TMA tensor-map encoding and kernel launches.  Nothing here allocates
// device memory; the only device state is the per-device error word.
#include <math.h>
#include <mutex>
#include <string.h>

#include "attn.h"
#include "kernels.h"

namespace attn {
namespace {

__device__ unsigned int g_error_word;

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::once_flag once;
  int status = ATTN_OK;            // ATTN_OK, ATTN_E_DEVICE or ATTN_E_CUDA
  unsigned int *err = nullptr;     // device address of g_error_word
};
DeviceState g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

// Per-device set-up: capability check and the error word's device address.
int device_state(unsigned int **err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_E_CUDA;
  DeviceState &s = g_dev[dev];
  std::call_once(s.once, [&s, dev] {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      s.status = ATTN_E_CUDA;
      return;
    }
    if (major != 10) {
      s.status = ATTN_E_DEVICE;
      return;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) {
      s.status = ATTN_E_CUDA;
      return;
    }
    s.err = static_cast<unsigned int *>(p);
  });
  *err = s.err;
  return s.status;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 3-D bf16 tensor map over a [rows, heads, d] row-major tensor: dims
// (d, heads, rows), box (64, 1, box_rows), 128-byte swizzle.
int encode_3d(CUtensorMap *map, const void *ptr, int d, int heads, long long rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return ATTN_E_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * heads * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_E_CUDA;
}

int check_threshold(float thr) {
  if (!(thr >= 0.f && thr <= 1.f)) return ATTN_E_THRESHOLD;   // also rejects NaN
  return ATTN_OK;
}

float thr_to_log2(float thr) {
  return thr > 0.f ? (float)log2((double)thr) : -INFINITY;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

int attn_get_config(attn_config *cfg) {
  if (!cfg) return ATTN_E_NULL;
  cfg->prefill_block_m = kPrefillBlockM;
  cfg->prefill_block_n = kPrefillBlockN;
  cfg->skip_tile = kSkipTile;
  cfg->decode_splits = kDecodeSplits;
  cfg->decode_split_tile = kDecodeSplitTile;
  cfg->decode_page_size = kPageSize;
  cfg->smallseq_max_s_kv = kSmallSeqMaxKv;
  return ATTN_OK;
}

const char *attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_E_NULL: return "ATTN_E_NULL";
    case ATTN_E_ALIGN: return "ATTN_E_ALIGN";
    case ATTN_E_HEADS: return "ATTN_E_HEADS";
    case ATTN_E_HEAD_DIM: return "ATTN_E_HEAD_DIM";
    case ATTN_E_THRESHOLD: return "ATTN_E_THRESHOLD";
    case ATTN_E_PAGE_SIZE: return "ATTN_E_PAGE_SIZE";
    case ATTN_E_SMALLSEQ: return "ATTN_E_SMALLSEQ";
    case ATTN_E_SHAPE: return "ATTN_E_SHAPE";
    case ATTN_E_WORKSPACE: return "ATTN_E_WORKSPACE";
    case ATTN_E_SCALE: return "ATTN_E_SCALE";
    case ATTN_E_CUDA: return "ATTN_E_CUDA";
    case ATTN_E_DEVICE: return "ATTN_E_DEVICE";
    case ATTN_E_TOO_LARGE: return "ATTN_E_TOO_LARGE";
    case ATTN_E_QDQ: return "ATTN_E_QDQ";
    default: return "ATTN_E_UNKNOWN";
  }
}

int attn_varlen_fwd_ex(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                       const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                       int batch, int total_q, int total_k, int max_q, int max_k,
                       int h_q, int h_kv, int d, int causal, float scale,
                       float skip_threshold, uint32_t *skip_mask,
                       unsigned long long *skip_counts,
                       attn_bf16 *out, float *lse, attn_stream_t stream) {
  if (batch < 0 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0) return ATTN_E_SHAPE;
  if (h_q < 1 || h_kv < 1 || h_q % h_kv != 0) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  int rc = check_threshold(skip_threshold);
  if (rc) return rc;
  if (batch > 0 && (max_q <= 0 || total_q <= 0)) return ATTN_E_SHAPE;
  if (!q || !k || !v || !cu_seqlens_q || !cu_seqlens_k || !out) return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_E_ALIGN;
  if ((long long)max_q > (1ll << 24) || (long long)max_k > (1ll << 24)) return ATTN_E_TOO_LARGE;
  unsigned int *err = nullptr;
  rc = device_state(&err);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  PrefillParams p{};
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.out = out;
  p.lse = lse;
  p.skip_mask = skip_mask;
  p.skip_counts = skip_counts;
  p.batch = batch;
  p.total_q = total_q;
  p.total_k = total_k;
  p.max_q = max_q;
  p.max_k = max_k;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = h_q / h_kv;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.qb_max = (max_q + kPrefillBlockM - 1) / kPrefillBlockM;
  p.kt_max = (max_k + kSkipTile - 1) / kSkipTile;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.thr_log2 = thr_to_log2(skip_threshold);
  p.err = err;
  // keys beyond the queries (chunked prefill): a sequence's items together
  p.seq_major = max_k > max_q ? 1 : 0;

  if (skip_mask) {
    const size_t bits = (size_t)batch * p.qb_max * h_q * p.kt_max;
    if (bits && cudaMemsetAsync(skip_mask, 0, align_up(bits, 32) / 8, st) != cudaSuccess)
      return ATTN_E_CUDA;
  }
  if (skip_counts && cudaMemsetAsync(skip_counts, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    return ATTN_E_CUDA;
  if (batch == 0) return ATTN_OK;

  CUtensorMap qmap, kmap, vmap, omap;
  if (encode_3d(&qmap, q, d, h_q, total_q, kPrefillBlockM) ||
      encode_3d(&kmap, k, d, h_kv, total_k, kPrefillBlockN) ||
      encode_3d(&vmap, v, d, h_kv, total_k, kPrefillBlockN) ||
      encode_3d(&omap, out, d, h_q, total_q, kPrefillBlockM))
    return ATTN_E_CUDA;
  return launch_prefill(p, qmap, kmap, vmap, omap, st) == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}

size_t attn_varlen_bwd_workspace_size(int total_q, int h_q) {
  if (total_q <= 0 || h_q <= 0) return 256;
  return align_up((size_t)total_q * h_q * sizeof(float), 256);
}

int attn_varlen_bwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v, const attn_bf16 *out,
                    const attn_bf16 *dout, const float *lse, const int32_t *cu_seqlens_q,
                    const int32_t *cu_seqlens_k, int batch, int total_q, int total_k, int max_q, int max_k,
                    int h_q, int h_kv, int d, int causal, float scale, attn_bf16 *dq, attn_bf16 *dk,
                    attn_bf16 *dv, void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  if (batch < 0 || total_q < 0 || total_k < 0 || max_q < 0 || max_k < 0) return ATTN_E_SHAPE;
  if (h_q < 1 || h_kv < 1 || h_q % h_kv != 0) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  if (batch > 0 && (max_q <= 0 || total_q <= 0)) return ATTN_E_SHAPE;
  if (!q || !k || !v || !out || !dout || !lse || !cu_seqlens_q || !cu_seqlens_k || !dq || !dk || !dv)
    return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_E_ALIGN;
  if ((long long)max_q > (1ll << 24) || (long long)max_k > (1ll << 24)) return ATTN_E_TOO_LARGE;
  // one CTA per (query block or key tile, head, sequence): the grids must fit 2^31 - 1
  if ((long long)batch * h_q * ((max_q + kPrefillBlockM - 1) / kPrefillBlockM) >= (1ll << 31) ||
      (long long)batch * h_kv * ((max_k + kPrefillBlockN - 1) / kPrefillBlockN) >= (1ll << 31))
    return ATTN_E_TOO_LARGE;
  if (batch > 0) {
    if (!workspace) return ATTN_E_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_E_ALIGN;
    if (workspace_bytes < attn_varlen_bwd_workspace_size(total_q, h_q)) return ATTN_E_WORKSPACE;
  }
  unsigned int *err = nullptr;
  int rc = device_state(&err);
  if (rc) return rc;
  if (batch == 0) return ATTN_OK;
  BwdParams p{};
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.delta = static_cast<float *>(workspace);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.batch = batch;
  p.total_q = total_q;
  p.total_k = total_k;
  p.max_q = max_q;
  p.max_k = max_k;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = h_q / h_kv;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.qb_max = (max_q + kPrefillBlockM - 1) / kPrefillBlockM;
  p.kt_max = (max_k + kPrefillBlockN - 1) / kPrefillBlockN;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  CUtensorMap qmap, kmap, vmap, dmap;
  if (encode_3d(&qmap, q, d, h_q, total_q, kPrefillBlockM) ||
      encode_3d(&kmap, k, d, h_kv, total_k, kPrefillBlockN) ||
      encode_3d(&vmap, v, d, h_kv, total_k, kPrefillBlockN) ||
      encode_3d(&dmap, dout, d, h_q, total_q, kPrefillBlockM))
    return ATTN_E_CUDA;
  return launch_backward(p, qmap, kmap, vmap, dmap, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? ATTN_OK
             : ATTN_E_CUDA;
}

int attn_paged_prefill(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                       const int32_t *block_table, const int32_t *cu_seqlens_q, const int32_t *seq_lens_k,
                       int batch, int total_q, int max_q, int max_k, int num_pages, int max_pages_per_seq,
                       int page_size, int h_q, int h_kv, int d, int causal, float scale,
                       float skip_threshold, uint32_t *skip_mask, unsigned long long *skip_counts,
                       attn_bf16 *out, float *lse, attn_stream_t stream) {
  if (batch < 0 || total_q < 0 || max_q < 0 || max_k < 0 || num_pages < 0 || max_pages_per_seq < 0)
    return ATTN_E_SHAPE;
  if (page_size != kPageSize) return ATTN_E_PAGE_SIZE;
  if (h_q < 1 || h_kv < 1 || h_q % h_kv != 0) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  int rc = check_threshold(skip_threshold);
  if (rc) return rc;
  if (batch > 0 && (max_q <= 0 || total_q <= 0 || num_pages <= 0 || max_pages_per_seq <= 0))
    return ATTN_E_SHAPE;
  if (!q || !k_cache || !v_cache || !block_table || !cu_seqlens_q || !seq_lens_k || !out) return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return ATTN_E_ALIGN;
  if ((long long)max_q > (1ll << 24) || (long long)max_k > (1ll << 24) ||
      (long long)num_pages * page_size > (1ll << 30) || (long long)max_pages_per_seq * page_size > (1ll << 30))
    return ATTN_E_TOO_LARGE;
  unsigned int *err = nullptr;
  rc = device_state(&err);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  PrefillParams p{};
  p.cu_q = cu_seqlens_q;
  p.out = out;
  p.lse = lse;
  p.skip_mask = skip_mask;
  p.skip_counts = skip_counts;
  p.batch = batch;
  p.total_q = total_q;
  p.max_q = max_q;
  p.max_k = max_k;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = h_q / h_kv;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.qb_max = (max_q + kPrefillBlockM - 1) / kPrefillBlockM;
  p.kt_max = (max_k + kSkipTile - 1) / kSkipTile;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.thr_log2 = thr_to_log2(skip_threshold);
  p.err = err;
  // keys beyond the queries (chunked prefill): a sequence's items together
  p.seq_major = max_k > max_q ? 1 : 0;
  p.paged = 1;
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.block_table = block_table;
  p.seq_lens_k = seq_lens_k;

  if (skip_mask) {
    const size_t bits = (size_t)batch * p.qb_max * h_q * p.kt_max;
    if (bits && cudaMemsetAsync(skip_mask, 0, align_up(bits, 32) / 8, st) != cudaSuccess)
      return ATTN_E_CUDA;
  }
  if (skip_counts && cudaMemsetAsync(skip_counts, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    return ATTN_E_CUDA;
  if (batch == 0) return ATTN_OK;

  CUtensorMap qmap, kmap, vmap, omap;
  const long long slots = (long long)num_pages * page_size;
  if (encode_3d(&qmap, q, d, h_q, total_q, kPrefillBlockM) ||
      encode_3d(&kmap, k_cache, d, h_kv, slots, kPageSize) ||
      encode_3d(&vmap, v_cache, d, h_kv, slots, kPageSize) ||
      encode_3d(&omap, out, d, h_q, total_q, kPrefillBlockM))
    return ATTN_E_CUDA;
  return launch_prefill(p, qmap, kmap, vmap, omap, st) == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}

int attn_varlen_fwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                    int batch, int total_q, int total_k, int max_q, int max_k,
                    int h_q, int h_kv, int d, int causal, float scale,
                    attn_bf16 *out, float *lse, attn_stream_t stream) {
  return attn_varlen_fwd_ex(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_q,
                            max_k, h_q, h_kv, d, causal, scale, 0.f, nullptr, nullptr, out, lse,
                            stream);
}

size_t attn_paged_decode_workspace_size(int batch, int h_q, int d) {
  if (batch <= 0 || h_q <= 0 || d <= 0) return 256;
  const size_t rows = (size_t)batch * h_q * kDecodeSplits;
  return align_up(rows * d * sizeof(float), 256) + align_up(rows * 2 * sizeof(float), 256);
}

}  // extern "C"

namespace {

// Two-pass skip-mode workspace: the split partials, then the scores
// [B, h_kv, s_stride, G], the 32-key tile maxima [B, h_kv, kt_max, G] and the
// split maxima [B, h_kv, splits, G] (all fp32).
struct SkipWorkspace {
  size_t o, ml, s, tmax, smax, total;
  int s_stride, kt_max;
};

SkipWorkspace skip_workspace(int batch, int h_q, int d, int max_pages_per_seq) {
  SkipWorkspace w{};
  const size_t rows = (size_t)batch * h_q * kDecodeSplits;
  const long long keys = (long long)max_pages_per_seq * kPageSize;
  w.s_stride = (int)((keys + 63) / 64 * 64);   // whole 64-key chunks
  w.kt_max = (int)((keys + kSkipTile - 1) / kSkipTile);
  w.o = 0;
  w.ml = w.o + align_up(rows * d * sizeof(float), 256);
  w.s = w.ml + align_up(rows * 2 * sizeof(float), 256);
  w.tmax = w.s + align_up((size_t)batch * h_q * w.s_stride * sizeof(float), 256);
  w.smax = w.tmax + align_up((size_t)batch * h_q * w.kt_max * sizeof(float), 256);
  w.total = w.smax + align_up(rows * sizeof(float), 256);
  return w;
}

// Host-checkable arguments of the paged decode entry points (everything but
// the workspace), in the order their error codes are documented.
int check_decode_args(const void *q, const void *k_cache, const void *v_cache, const void *block_table,
                      const void *seq_lens, int batch, int num_pages, int max_pages_per_seq, int page_size,
                      int h_q, int h_kv, int d, float skip_threshold, float scale, const void *out) {
  if (batch < 0 || num_pages < 0 || max_pages_per_seq < 0) return ATTN_E_SHAPE;
  if (page_size != kPageSize) return ATTN_E_PAGE_SIZE;
  if (h_q < 1 || h_kv < 1 || h_q % h_kv != 0 || h_q / h_kv > kMaxGroup) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  const int rc = check_threshold(skip_threshold);
  if (rc) return rc;
  if (batch > 0 && (num_pages <= 0 || max_pages_per_seq <= 0)) return ATTN_E_SHAPE;
  if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !out) return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return ATTN_E_ALIGN;
  if ((long long)max_pages_per_seq * page_size > (1ll << 30)) return ATTN_E_TOO_LARGE;
  return ATTN_OK;
}

}  // namespace

extern "C" {

size_t attn_paged_decode_workspace_size_ex(int batch, int h_q, int d, int max_pages_per_seq,
                                           float skip_threshold) {
  if (!(skip_threshold > 0.f)) return attn_paged_decode_workspace_size(batch, h_q, d);
  if (batch <= 0 || h_q <= 0 || d <= 0 || max_pages_per_seq <= 0) return 256;
  return skip_workspace(batch, h_q, d, max_pages_per_seq).total;
}

}  // extern "C"

namespace {

// NVFP4 quantise-dequantise of the decode's P and V (see attn.h).
struct QdqSpec {
  bool p, v;
  float p_amax, v_amax;
};

// 448 / amax, and the ratio table g / (1 + j / 8), g = 2688 / amax (fp32).
void qdq_constants(float amax, float *k, float *tab) {
  *k = 448.0f / amax;
  const float g = 2688.0f / amax;
  for (int j = 0; j < 8; ++j) tab[j] = g / (1.0f + (float)j / 8.0f);
}

int paged_decode_impl(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                      const int32_t *block_table, const int32_t *seq_lens, int batch, int num_pages,
                      int max_pages_per_seq, int page_size, int h_q, int h_kv, int d, float skip_threshold,
                      float scale, const QdqSpec *qdq, uint32_t *skip_mask, unsigned long long *skip_counts,
                      attn_bf16 *out, float *lse, void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  int rc = check_decode_args(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages,
                             max_pages_per_seq, page_size, h_q, h_kv, d, skip_threshold, scale, out);
  if (rc) return rc;
  const bool quant = qdq && (qdq->p || qdq->v);
  // the 32-key skip schedules: skip-softmax on, or P / V quantised (at any threshold)
  const bool skip = skip_threshold > 0.f || quant;
  // skip mode: two passes over the split schedule with a workspace, one
  // sequential split per (sequence, kv-head) without
  const bool two_pass = skip && workspace != nullptr;
  if ((!skip || two_pass) && batch > 0) {
    if (!workspace) return ATTN_E_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_E_ALIGN;
    const size_t need = skip ? skip_workspace(batch, h_q, d, max_pages_per_seq).total
                             : attn_paged_decode_workspace_size(batch, h_q, d);
    if (workspace_bytes < need) return ATTN_E_WORKSPACE;
  }
  unsigned int *err = nullptr;
  rc = device_state(&err);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  DecodeParams p{};
  p.q = q;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = out;
  p.lse = lse;
  const size_t rows = (size_t)batch * h_q * kDecodeSplits;
  p.ws_o = static_cast<float *>(workspace);
  p.ws_ml = workspace ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                   align_up(rows * d * sizeof(float), 256))
                      : nullptr;
  p.skip_mask = skip_mask;
  p.skip_counts = skip_counts;
  p.batch = batch;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = h_q / h_kv;
  p.d = d;
  p.num_pages = num_pages;
  p.max_pages = max_pages_per_seq;
  p.kt_max = (max_pages_per_seq * page_size + kSkipTile - 1) / kSkipTile;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.thr_log2 = thr_to_log2(skip_threshold);
  p.sequential = skip ? (two_pass ? 2 : 1) : 0;
  if (quant) {
    p.p_qdq = qdq->p ? 1 : 0;
    p.v_qdq = qdq->v ? 1 : 0;
    float inv = 1.0f;
    if (qdq->p) {
      qdq_constants(qdq->p_amax, &p.p_k, p.p_tab);
      inv *= qdq->p_amax / 2688.0f;
    }
    if (qdq->v) {
      qdq_constants(qdq->v_amax, &p.v_k, p.v_tab);
      inv *= qdq->v_amax / 2688.0f;
    }
    p.qdq_out = inv;
  }
  size_t one_pass_clear = 0;   // bytes to zero at ws_s before a one-pass launch
  if (two_pass && batch > 0) {
    const SkipWorkspace w = skip_workspace(batch, h_q, d, max_pages_per_seq);
    char *base = static_cast<char *>(workspace);
    p.ws_o = reinterpret_cast<float *>(base + w.o);
    p.ws_ml = reinterpret_cast<float *>(base + w.ml);
    p.ws_s = reinterpret_cast<float *>(base + w.s);
    p.ws_tmax = reinterpret_cast<float *>(base + w.tmax);
    p.ws_smax = reinterpret_cast<float *>(base + w.smax);
    p.s_stride = w.s_stride;
    // Without quantisation, and when a split's scores fit in shared memory,
    // one pass replaces the two: each split's CTA keeps its scores on chip and
    // waits for the earlier splits' maxima.  Its ticket counter and published
    // maxima take the start of the scores area, zeroed before the launch.
    const long long n128 = ((long long)max_pages_per_seq * kPageSize + kDecodeSplitTile - 1) / kDecodeSplitTile;
    const int split_keys = (int)((n128 + kDecodeSplits - 1) / kDecodeSplits) * kDecodeSplitTile;
    const size_t pub_bytes = (size_t)batch * h_q * kDecodeSplits * sizeof(unsigned long long);
    if (!quant && decode_one_pass_smem(d, h_q / h_kv, split_keys) != 0 &&
        256 + pub_bytes <= w.tmax - w.s) {
      p.sequential = 3;
      p.split_keys = split_keys;
      p.ws_ticket = reinterpret_cast<unsigned int *>(base + w.s);
      p.ws_pub = reinterpret_cast<unsigned long long *>(base + w.s + 256);
      one_pass_clear = 256 + pub_bytes;
    }
  }
  p.err = err;

  if (skip_mask) {
    const size_t bits = (size_t)batch * h_kv * p.kt_max;
    if (bits && cudaMemsetAsync(skip_mask, 0, align_up(bits, 32) / 8, st) != cudaSuccess)
      return ATTN_E_CUDA;
  }
  if (skip_counts && cudaMemsetAsync(skip_counts, 0, 2 * sizeof(unsigned long long), st) != cudaSuccess)
    return ATTN_E_CUDA;
  if (batch == 0) return ATTN_OK;
  if (one_pass_clear && cudaMemsetAsync(p.ws_s, 0, one_pass_clear, st) != cudaSuccess) return ATTN_E_CUDA;

  CUtensorMap kmap, vmap;
  const long long slots = (long long)num_pages * page_size;
  if (encode_3d(&kmap, k_cache, d, h_kv, slots, kPageSize) ||
      encode_3d(&vmap, v_cache, d, h_kv, slots, kPageSize))
    return ATTN_E_CUDA;
  return launch_decode(p, kmap, vmap, st) == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}

}  // namespace

extern "C" {

int attn_paged_decode_ex(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                         const int32_t *block_table, const int32_t *seq_lens,
                         int batch, int num_pages, int max_pages_per_seq, int page_size,
                         int h_q, int h_kv, int d, float skip_threshold, float scale,
                         uint32_t *skip_mask, unsigned long long *skip_counts,
                         attn_bf16 *out, float *lse,
                         void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  return paged_decode_impl(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages, max_pages_per_seq,
                           page_size, h_q, h_kv, d, skip_threshold, scale, nullptr, skip_mask, skip_counts, out,
                           lse, workspace, workspace_bytes, stream);
}

size_t attn_paged_decode_qdq_workspace_size(int batch, int h_q, int d, int max_pages_per_seq) {
  return attn_paged_decode_workspace_size_ex(batch, h_q, d, max_pages_per_seq, 1.0f);
}

int attn_paged_decode_qdq(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                          const int32_t *block_table, const int32_t *seq_lens, int batch, int num_pages,
                          int max_pages_per_seq, int page_size, int h_q, int h_kv, int d, float skip_threshold,
                          float scale, int p_qdq, float p_qdq_amax, int v_qdq, float v_qdq_amax,
                          uint32_t *skip_mask, unsigned long long *skip_counts, attn_bf16 *out, float *lse,
                          void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  int rc = check_decode_args(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages, max_pages_per_seq,
                             page_size, h_q, h_kv, d, skip_threshold, scale, out);
  if (rc) return rc;
  auto amax_ok = [](float a) { return isfinite(a) && a >= 0x1p-64f && a <= 0x1p64f; };
  if ((p_qdq != ATTN_QDQ_NONE && p_qdq != ATTN_QDQ_NVFP4) || (v_qdq != ATTN_QDQ_NONE && v_qdq != ATTN_QDQ_NVFP4))
    return ATTN_E_QDQ;
  if ((p_qdq == ATTN_QDQ_NVFP4 && !amax_ok(p_qdq_amax)) || (v_qdq == ATTN_QDQ_NVFP4 && !amax_ok(v_qdq_amax)))
    return ATTN_E_QDQ;
  QdqSpec spec{p_qdq == ATTN_QDQ_NVFP4, v_qdq == ATTN_QDQ_NVFP4, p_qdq_amax, v_qdq_amax};
  return paged_decode_impl(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages, max_pages_per_seq,
                           page_size, h_q, h_kv, d, skip_threshold, scale, &spec, skip_mask, skip_counts, out,
                           lse, workspace, workspace_bytes, stream);
}

int attn_paged_decode(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                      const int32_t *block_table, const int32_t *seq_lens,
                      int batch, int num_pages, int max_pages_per_seq, int page_size,
                      int h_q, int h_kv, int d, float skip_threshold, float scale,
                      attn_bf16 *out, float *lse,
                      void *workspace, size_t workspace_bytes, attn_stream_t stream) {
  return attn_paged_decode_ex(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages,
                              max_pages_per_seq, page_size, h_q, h_kv, d, skip_threshold, scale,
                              nullptr, nullptr, out, lse, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace attn {
namespace {

// Scratch for attn_paged_decode_static: split-KV partials of callers that
// cannot allocate.  Shared by every call on a device; see attn.h.
static __device__ __align__(256) unsigned char g_static_workspace[ATTN_STATIC_WORKSPACE_BYTES];

struct StaticScratch {
  std::once_flag once;
  cudaError_t status = cudaSuccess;
  void *ptr = nullptr;
};
StaticScratch g_scratch[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device with that device current.  Host code must not pass the array's
// name itself to a kernel: on the host it is only a stand-in symbol.
int static_scratch(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_E_CUDA;
  StaticScratch &s = g_scratch[dev];
  std::call_once(s.once, [&s] {
    void *p = nullptr;
    s.status = cudaGetSymbolAddress(&p, g_static_workspace);
    s.ptr = (s.status == cudaSuccess) ? p : nullptr;
  });
  if (s.status != cudaSuccess || !s.ptr) return ATTN_E_CUDA;
  *ptr = s.ptr;
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

extern "C" {

int attn_paged_decode_static(const attn_bf16 *q, const attn_bf16 *k_cache, const attn_bf16 *v_cache,
                             const int32_t *block_table, const int32_t *seq_lens, int batch,
                             int num_pages, int max_pages_per_seq, int page_size, int h_q, int h_kv,
                             int d, float skip_threshold, float scale, attn_bf16 *out, float *lse,
                             attn_stream_t stream) {
  // the same argument checks (and error codes) as attn_paged_decode_ex
  int rc = check_decode_args(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages,
                             max_pages_per_seq, page_size, h_q, h_kv, d, skip_threshold, scale, out);
  if (rc) return rc;
  const bool skip = skip_threshold > 0.f;
  if (!skip && attn_paged_decode_workspace_size(batch, h_q, d) > ATTN_STATIC_WORKSPACE_BYTES)
    return ATTN_E_TOO_LARGE;
  unsigned int *err = nullptr;
  rc = device_state(&err);
  if (rc) return rc;
  void *scratch = nullptr;
  rc = static_scratch(&scratch);
  if (rc) return rc;
  // skip mode: the two-pass schedule when its workspace fits the scratch array,
  // else the sequential one, which needs none
  if (skip && attn_paged_decode_workspace_size_ex(batch, h_q, d, max_pages_per_seq, skip_threshold) >
                  ATTN_STATIC_WORKSPACE_BYTES)
    scratch = nullptr;
  return attn_paged_decode_ex(q, k_cache, v_cache, block_table, seq_lens, batch, num_pages,
                              max_pages_per_seq, page_size, h_q, h_kv, d, skip_threshold, scale,
                              nullptr, nullptr, out, lse, scratch, scratch ? ATTN_STATIC_WORKSPACE_BYTES : 0,
                              stream);
}

int attn_smallseq_fwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v,
                      const int32_t *cu_seqlens_kv, int batch, int total_kv, int h, int d,
                      int max_s_kv, float scale, attn_bf16 *out, attn_bf16 *weights,
                      attn_stream_t stream) {
  if (batch < 0 || total_kv < 0) return ATTN_E_SHAPE;
  if (h < 1) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (max_s_kv < 1 || max_s_kv > kSmallSeqMaxKv) return ATTN_E_SMALLSEQ;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  if (!q || !k || !v || !cu_seqlens_kv || !out) return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_E_ALIGN;
  if (weights && (reinterpret_cast<uintptr_t>(weights) & 1u)) return ATTN_E_ALIGN;
  unsigned int *err = nullptr;
  int rc = device_state(&err);
  if (rc) return rc;
  SmallSeqParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.cu = cu_seqlens_kv;
  p.out = out;
  p.weights = weights;
  p.batch = batch;
  p.total_kv = total_kv;
  p.h = h;
  p.d = d;
  p.max_s_kv = max_s_kv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  return launch_smallseq(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}

int attn_smallseq_bwd(const attn_bf16 *q, const attn_bf16 *k, const attn_bf16 *v, const attn_bf16 *dout,
                      const attn_bf16 *weights, const int32_t *cu_seqlens_kv, int batch, int total_kv,
                      int h, int d, int max_s_kv, float scale, attn_bf16 *dq, attn_bf16 *dk,
                      attn_bf16 *dv, attn_stream_t stream) {
  if (batch < 0 || total_kv < 0) return ATTN_E_SHAPE;
  if (h < 1) return ATTN_E_HEADS;
  if (d != 64 && d != 128) return ATTN_E_HEAD_DIM;
  if (max_s_kv < 1 || max_s_kv > kSmallSeqMaxKv) return ATTN_E_SMALLSEQ;
  if (!isfinite(scale) || !(scale > 0.f)) return ATTN_E_SCALE;
  if (!q || !k || !v || !dout || !weights || !cu_seqlens_kv || !dq || !dk || !dv) return ATTN_E_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return ATTN_E_ALIGN;
  if (reinterpret_cast<uintptr_t>(weights) & 1u) return ATTN_E_ALIGN;
  unsigned int *err = nullptr;
  int rc = device_state(&err);
  if (rc) return rc;
  SmallSeqParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.cu = cu_seqlens_kv;
  p.dout = dout;
  p.weights_in = weights;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.batch = batch;
  p.total_kv = total_kv;
  p.h = h;
  p.d = d;
  p.max_s_kv = max_s_kv;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = err;
  return launch_smallseq_bwd(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ATTN_OK : ATTN_E_CUDA;
}


int attn_get_last_device_error(attn_stream_t stream) {
  unsigned int *err = nullptr;
  int rc = device_state(&err);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_E_CUDA;
  unsigned int host = 0;
  if (cudaMemcpyFromSymbol(&host, g_error_word, sizeof(host)) != cudaSuccess) return ATTN_E_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return ATTN_E_CUDA;
  return (int)host;
}

}  // extern "C"
