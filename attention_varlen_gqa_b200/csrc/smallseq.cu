// smallseq.cu -- s_q = 1, s_kv <= 16 cross attention (sm_100a).
//
// ROCm/TransformerEngine PR 461 ("Integrate CK varlen cross attention for
// small-seq (s_q=1, s_kv<=16)") runs this case as three kernels (scores,
// mask + softmax, output) with runtime dispatch over max_seqlen_kv in
// {2,4,6,8,12,16}.  Here it is one fused, memory-bound kernel: each warp owns
// one (query token, head) row, keeps its <= 16 scores in registers, and
// reads q, the row's K and V exactly once with coalesced 256-byte row loads
// (lane i holds dims [D/32*i, D/32*(i+1))).  All K and V loads of a row are
// issued before the first reduction so a warp keeps up to 2*NK row loads in
// flight; many warps per SM cover HBM latency.  Batch = number of query
// tokens (the page's b_varlen = max_tokens_q reading).
#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kThreads = 128;   // 4 warps per CTA, one (token, head) row per warp at a time

template <int D>
struct RowVec;
template <>
struct RowVec<128> {          // 4 bf16 per lane
  using T = uint2;
  static constexpr int E = 4;
};
template <>
struct RowVec<64> {           // 2 bf16 per lane
  using T = uint32_t;
  static constexpr int E = 2;
};

ATTN_DEVICE void unpack(const uint2 &x, float *f) {
  f[0] = bf16_lo(x.x); f[1] = bf16_hi(x.x); f[2] = bf16_lo(x.y); f[3] = bf16_hi(x.y);
}
ATTN_DEVICE void unpack(const uint32_t &x, float *f) { f[0] = bf16_lo(x); f[1] = bf16_hi(x); }

ATTN_DEVICE uint2 ldg_stream(const uint2 *p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
ATTN_DEVICE uint32_t ldg_stream(const uint32_t *p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

template <int D>
ATTN_DEVICE void store_row(uint16_t *dst, const float *o);
template <>
ATTN_DEVICE void store_row<128>(uint16_t *dst, const float *o) {
  uint2 w = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
  *reinterpret_cast<uint2 *>(dst) = w;
}
template <>
ATTN_DEVICE void store_row<64>(uint16_t *dst, const float *o) {
  *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(o[0], o[1]);
}

// NK: key bucket (the smallest of {2,4,6,8,12,16} >= max_s_kv).
template <int D, int NK>
__global__ void __launch_bounds__(kThreads, 4) smallseq_kernel(SmallSeqParams p) {
  using V = typename RowVec<D>::T;
  constexpr int E = RowVec<D>::E;
  const int lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  const long long units = (long long)p.batch * p.h;
  const long long stride = (long long)gridDim.x * warps_per_cta;

  for (long long u = (long long)blockIdx.x * warps_per_cta + (threadIdx.x >> 5); u < units;
       u += stride) {
    const int b = int(u / p.h);
    const int hh = int(u - (long long)b * p.h);
    const int k0 = __ldg(p.cu + b);
    const int k1 = __ldg(p.cu + b + 1);
    const int n = k1 - k0;
    uint16_t *orow = p.out + (size_t)u * D + lane * E;
    uint16_t *wrow = p.weights ? p.weights + (size_t)u * p.max_s_kv : nullptr;

    bool bad = (k0 < 0) | (n < 0) | (k1 > p.total_kv);
    bool too_long = (!bad) & (n > p.max_s_kv);
    if (bad | too_long | (n == 0)) {
      if (lane == 0) {
        if (bad) raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
        if (too_long) raise_error(p.err, ATTN_DEVERR_SMALLSEQ_LEN);
      }
      float z[E] = {};
      store_row<D>(orow, z);
      if (wrow && lane < p.max_s_kv) wrow[lane] = 0;
      continue;
    }

    // q row and all key / value rows of this (token, head)
    const V qv = ldg_stream(reinterpret_cast<const V *>(p.q + (size_t)u * D) + lane);
    V kr[NK], vr[NK];
    const size_t row_stride = (size_t)p.h * D;
    const V *kb = reinterpret_cast<const V *>(p.k + (size_t)k0 * row_stride + (size_t)hh * D) + lane;
    const V *vb = reinterpret_cast<const V *>(p.v + (size_t)k0 * row_stride + (size_t)hh * D) + lane;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < n) {
        kr[j] = ldg_stream(kb + (size_t)j * (row_stride / E));
        vr[j] = ldg_stream(vb + (size_t)j * (row_stride / E));
      }
    }
    float qf[E];
    unpack(qv, qf);

    // scores (log2 domain), reduced across the warp; every lane ends with all
    float s[NK];
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < n) {
        float kf[E];
        unpack(kr[j], kf);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc = fmaf(qf[e], kf[e], acc);
        s[j] = warp_sum(acc) * p.scale_log2;
      } else {
        s[j] = -INFINITY;
      }
    }
    float m = s[0];
#pragma unroll
    for (int j = 1; j < NK; ++j) m = fmaxf(m, s[j]);
    float l = 0.f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      s[j] = (j < n) ? ex2(s[j] - m) : 0.f;
      l += s[j];
    }
    const float inv = 1.f / l;

    float o[E] = {};
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (j < n) {
        float vf[E];
        unpack(vr[j], vf);
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(s[j], vf[e], o[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] *= inv;
    store_row<D>(orow, o);

    if (wrow) {
      float w = 0.f;
#pragma unroll
      for (int j = 0; j < NK; ++j)
        if (lane == j) w = s[j] * inv;
      if (lane < p.max_s_kv) wrow[lane] = f32_to_bf16(w);
    }
  }
}

template <int D, int NK>
cudaError_t launch_nk(const SmallSeqParams &p, cudaStream_t stream) {
  static int blocks_per_sm = 0;
  static int num_sms = 0;
  if (blocks_per_sm == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, smallseq_kernel<D, NK>, kThreads, 0);
    if (blocks_per_sm < 1) blocks_per_sm = 1;
  }
  const long long units = (long long)p.batch * p.h;
  long long want = (units + kThreads / 32 - 1) / (kThreads / 32);
  long long cap = (long long)num_sms * blocks_per_sm;
  int grid = int(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  smallseq_kernel<D, NK><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const SmallSeqParams &p, cudaStream_t stream) {
  const int m = p.max_s_kv;
  if (m <= 2) return launch_nk<D, 2>(p, stream);
  if (m <= 4) return launch_nk<D, 4>(p, stream);
  if (m <= 6) return launch_nk<D, 6>(p, stream);
  if (m <= 8) return launch_nk<D, 8>(p, stream);
  if (m <= 12) return launch_nk<D, 12>(p, stream);
  return launch_nk<D, 16>(p, stream);
}

}  // namespace

cudaError_t launch_smallseq(const SmallSeqParams &p, cudaStream_t stream) {
  if ((long long)p.batch * p.h == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128>(p, stream) : launch_d<64>(p, stream);
}

}  // namespace attn
