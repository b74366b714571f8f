// smallseq.cu -- s_q = 1, s_kv <= 16 cross attention (sm_100a).
//
// ROCm/TransformerEngine PR 461 ("Integrate CK varlen cross attention for
// small-seq (s_q=1, s_kv<=16)") runs this case as three kernels (scores,
// mask + softmax, output) with runtime dispatch over max_seqlen_kv in
// {2,4,6,8,12,16}; the batch counts query tokens.  Here it is one fused,
// memory-bound kernel.
//
// One warp per (query token, head) row, lane i holding dims [d/32 i,
// d/32 (i + 1)) so every row load is one coalesced 256-byte transaction.  The
// row's own key count picks the code path (up to 4, 8 or 16 keys), so no
// work is spent on absent keys; all K and V loads of a row are issued before
// the first use (128 registers a thread, 16 warps per SM: measured faster than
// 24 or 32 warps with fewer loads in flight each).  The <= 16 partial dot products are reduced across
// the warp by a reduce-scatter shuffle tree (16 shuffles for 16 keys instead
// of 80); softmax, weights and O = P V stay in registers.  Measured against a
// shared-memory ring fed by bulk or cp.async copies: 3.5 TB/s here vs 1.2-1.3
// TB/s there (one 198 KB CTA per SM left too few warps for the compute).
#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;

template <int D>
struct LaneVec;
template <>
struct LaneVec<128> {   // 4 bf16 per lane
  using T = uint2;
  static constexpr int E = 4;
  static ATTN_DEVICE void unpack(const T &x, float *f) {
    f[0] = bf16_lo(x.x); f[1] = bf16_hi(x.x); f[2] = bf16_lo(x.y); f[3] = bf16_hi(x.y);
  }
  static ATTN_DEVICE T pack(const float *f) { return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3])); }
};
template <>
struct LaneVec<64> {    // 2 bf16 per lane
  using T = uint32_t;
  static constexpr int E = 2;
  static ATTN_DEVICE void unpack(const T &x, float *f) { f[0] = bf16_lo(x); f[1] = bf16_hi(x); }
  static ATTN_DEVICE T pack(const float *f) { return pack_bf16x2(f[0], f[1]); }
};

// One halving step of the reduce-scatter: of the CNT values left, keep the
// half whose key bit matches this lane's bit STEP and add the partner's copy.
template <int NK, int CNT>
ATTN_DEVICE void rs_step(float (&a)[NK], int lane) {
  if constexpr (CNT > 1) {
    constexpr int H = CNT / 2;
    constexpr int STEP = 16 * CNT / NK;
    const bool hi = (lane & STEP) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float keep = hi ? a[H + i] : a[i];
      const float send = hi ? a[i] : a[H + i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, STEP);
    }
    rs_step<NK, H>(a, lane);
  }
}

// Sum of v[0..NK) over the 32 lanes, scattered: afterwards lane l holds the
// full sum of key (l >> S) with S = log2(32 / NK) (each key in 32 / NK lanes).
template <int NK>
ATTN_DEVICE float reduce_scatter(float (&v)[NK], int lane) {
  rs_step<NK, NK>(v, lane);
  float s = v[0];
  // the lane bits below the key bits still hold partial sums of the same key
#pragma unroll
  for (int step = 32 / NK / 2; step >= 1; step >>= 1) s += __shfl_xor_sync(0xffffffffu, s, step);
  return s;
}

ATTN_DEVICE uint2 ldg_stream(const uint2 *p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
ATTN_DEVICE uint32_t ldg_stream(const uint32_t *p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

// One (query token, head) row with n <= NK keys.  V_WITH_K: issue the V
// loads together with the K loads (more bytes in flight, more registers).
template <int D, int NK, bool V_WITH_K>
ATTN_DEVICE void row_attention(const SmallSeqParams &p, long long u, int hh, int k0, int n, int lane) {
  using LV = LaneVec<D>;
  using T = typename LV::T;
  constexpr int E = LV::E;
  static_assert(NK == 4 || NK == 8 || NK == 16, "power-of-two key counts for the reduce-scatter");
  constexpr int SH = (NK == 16) ? 1 : (NK == 8) ? 2 : 3;  // key of lane l after the reduce-scatter is l >> SH
  const size_t stride = (size_t)p.h * D / E;           // one key in units of T
  const T *kb = reinterpret_cast<const T *>(p.k + ((size_t)k0 * p.h + hh) * D) + lane;
  const T *vb = reinterpret_cast<const T *>(p.v + ((size_t)k0 * p.h + hh) * D) + lane;
  const T qv = ldg_stream(reinterpret_cast<const T *>(p.q + (size_t)u * D) + lane);
  T kr[NK], vr[V_WITH_K ? NK : 1];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    if (j < n) {
      kr[j] = ldg_stream(kb + j * stride);
      if (V_WITH_K) vr[j] = ldg_stream(vb + j * stride);
    }
  }
  float q[E];
  LV::unpack(qv, q);
  float part[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    float kf[E];
    LV::unpack(kr[j], kf);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc = fmaf(q[e], kf[e], acc);
    part[j] = (j < n) ? acc : 0.f;
  }
  const int key = lane >> SH;
  const float sc = reduce_scatter<NK>(part, lane);
  const float s2 = (key < n) ? sc * p.scale_log2 : -INFINITY;
  const float m = warp_max(s2);
  const float pr = (key < n) ? ex2(s2 - m) : 0.f;
  const float l = warp_sum(((lane & ((1 << SH) - 1)) == 0) ? pr : 0.f);
  const float inv = 1.f / l;
  float o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] = 0.f;
  if (V_WITH_K) {
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const float pj = __shfl_sync(0xffffffffu, pr, j << SH);
      if (j < n) {
        float vf[E];
        LV::unpack(vr[j], vf);
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(pj, vf[e], o[e]);
      }
    }
  } else {
    T vr2[NK];
#pragma unroll
    for (int j = 0; j < NK; ++j)
      if (j < n) vr2[j] = ldg_stream(vb + j * stride);
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const float pj = __shfl_sync(0xffffffffu, pr, j << SH);
      if (j < n) {
        float vf[E];
        LV::unpack(vr2[j], vf);
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(pj, vf[e], o[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] *= inv;
  reinterpret_cast<T *>(p.out + (size_t)u * D)[lane] = LV::pack(o);
  if (p.weights) {
    const float pt = __shfl_sync(0xffffffffu, pr, (lane < NK ? lane : 0) << SH);
    if (lane < p.max_s_kv) p.weights[(size_t)u * p.max_s_kv + lane] = f32_to_bf16(lane < n ? pt * inv : 0.f);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 4) smallseq_kernel(SmallSeqParams p) {
  using LV = LaneVec<D>;
  const int lane = threadIdx.x & 31;
  const long long units = (long long)p.batch * p.h;
  const long long stride = (long long)gridDim.x * kWarps;
  for (long long u = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5); u < units; u += stride) {
    const int b = (int)(u / p.h);
    const int hh = (int)(u - (long long)b * p.h);
    const int k0 = __ldg(p.cu + b), k1 = __ldg(p.cu + b + 1);
    const int n = k1 - k0;
    const bool bad = (k0 < 0) | (n < 0) | (k1 > p.total_kv);
    const bool too_long = !bad && n > p.max_s_kv;
    if (bad | too_long | (n == 0)) {
      if (lane == 0) {
        if (bad) raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
        if (too_long) raise_error(p.err, ATTN_DEVERR_SMALLSEQ_LEN);
      }
      float z[LV::E] = {};
      reinterpret_cast<typename LV::T *>(p.out + (size_t)u * D)[lane] = LV::pack(z);
      if (p.weights && lane < p.max_s_kv) p.weights[(size_t)u * p.max_s_kv + lane] = 0;
      continue;
    }
    if (n <= 4)
      row_attention<D, 4, true>(p, u, hh, k0, n, lane);
    else if (n <= 8)
      row_attention<D, 8, true>(p, u, hh, k0, n, lane);
    else
      row_attention<D, 16, true>(p, u, hh, k0, n, lane);
  }
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
  }
  return n;
}

template <int D>
cudaError_t launch_d(const SmallSeqParams &p, cudaStream_t stream) {
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, smallseq_kernel<D>, kThreads, 0);
  if (per_sm < 1) per_sm = 1;
  const long long rows = (long long)p.batch * p.h;
  const long long want = (rows + kWarps - 1) / kWarps;
  const long long cap = (long long)num_sms() * per_sm;
  const int grid = (int)(want < cap ? want : cap);
  smallseq_kernel<D><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_smallseq(const SmallSeqParams &p, cudaStream_t stream) {
  if ((long long)p.batch * p.h == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128>(p, stream) : launch_d<64>(p, stream);
}

}  // namespace attn
