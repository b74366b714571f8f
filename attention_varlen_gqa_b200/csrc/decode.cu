// decode.cu -- paged one-token decode with split-KV + LSE combine, and the
// sequential skip-softmax schedule (sm_100a).
//
// NVIDIA/Model-Optimizer PR 1941 ("Add split-k decode kernel for skip
// softmax"), What does this PR do?:
//   * skip-softmax off: the 32-split schedule of 128-token tiles, followed by
//     a log-sum-exp combine of the split partials;
//   * skip-softmax on: one sequential KV split per (sequence, kv-head) with
//     32-token tiles, so every decision sees the running softmax maximum;
//   * the threshold is a runtime argument.
//
// One CTA = one (sequence b, kv-head hk, split) with one warp per query head
// of the GQA group (G warps).  K and V pages are gathered through the block
// table with 3-D TMA copies (box = 64 dims x 1 head x 16 tokens, 128-byte
// swizzle) into shared-memory rings.  The loop runs two passes over 32-token
// tiles that are kLookahead tiles apart:
//   score pass (tile i):  S = q.K^T for all G heads (warp = head, lane =
//       token), tile max, skip vote of every head, running max.  The V copy
//       of tile i is only issued when the tile is kept.
//   PV pass (tile i - kLookahead): online-softmax rescale and O += P V.
// For thresholds <= 1 a skipped tile never raises a row's running max, so
// the decisions only need the K tiles: V copies get kLookahead tiles of
// latency cover and skipped tiles cost no V traffic at all.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kTile = 32;               // tokens per internal tile (skip unit)
constexpr int kKStages = 4;             // K ring depth
constexpr int kLookahead = 3;           // PV pass lags the score pass by this many tiles
constexpr int kVStages = kLookahead + 1;
constexpr int kRing = kLookahead + 1;   // score ring
static_assert(kDecodeSplits == 32, "the combine kernel gives one lane per split");
static_assert(kLookahead < 32, "kept flags live in one 32-bit word");

template <int D>
struct DecodeLayout {
  static constexpr int kSlot = kTile * D * 2;        // bytes of one K or V tile
  static constexpr int kBoxBytes = 16 * 64 * 2;      // one TMA box: 16 tokens x 64 dims
  static constexpr int kHalves = D / 64;
  static constexpr int kEPL = D / 32;                // dims per lane in the PV pass
  static size_t bytes(int G) {
    return 1024 + (size_t)(kKStages + kVStages) * kSlot + (size_t)G * D * 4 +
           (size_t)kRing * G * 32 * 4 * 2 + (kKStages + kVStages) * 8;
  }
};

ATTN_DEVICE uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D>
ATTN_DEVICE void pv_load(const uint8_t *slot, int t, int lane, float *v);
template <>
ATTN_DEVICE void pv_load<128>(const uint8_t *slot, int t, int lane, float *v) {
  const int half = lane >> 4, chunk = (lane & 15) >> 1;
  const uint2 x = *reinterpret_cast<const uint2 *>(slot + half * 4096 + sw128_offset(t, chunk) +
                                                   (lane & 1) * 8);
  v[0] = bf16_lo(x.x); v[1] = bf16_hi(x.x); v[2] = bf16_lo(x.y); v[3] = bf16_hi(x.y);
}
template <>
ATTN_DEVICE void pv_load<64>(const uint8_t *slot, int t, int lane, float *v) {
  const int chunk = lane >> 2;
  const uint32_t x = *reinterpret_cast<const uint32_t *>(slot + sw128_offset(t, chunk) + (lane & 3) * 4);
  v[0] = bf16_lo(x); v[1] = bf16_hi(x);
}

template <int D>
__global__ void __launch_bounds__(512, 1) decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                                     const __grid_constant__ CUtensorMap vmap,
                                                     DecodeParams p) {
  using Lay = DecodeLayout<D>;
  constexpr int E = Lay::kEPL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const int G = p.group;
  const int nthr = G * 32;
  uint8_t *ks_base = base;
  uint8_t *vs_base = base + kKStages * Lay::kSlot;
  float *q_s = reinterpret_cast<float *>(vs_base + kVStages * Lay::kSlot);     // [G][D]
  float *s_ring = q_s + G * D;                                                 // [kRing][G*32]
  float *tm_ring = s_ring + kRing * nthr;                                      // [kRing][G*32]
  uint64_t *kfull = reinterpret_cast<uint64_t *>(tm_ring + kRing * nthr);
  uint64_t *vfull = kfull + kKStages;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int hq = hk * G + w;
  const int nsplit = gridDim.x;

  int L = __ldg(p.seq_lens + b);
  const bool bad_len = (L < 0) | (L > p.max_pages * kPageSize);
  if (bad_len) L = 0;
  const int n_tiles = (L + kTile - 1) / kTile;
  int t0 = 0, t1 = n_tiles;
  if (!p.sequential) {
    const int n128 = (L + kDecodeSplitTile - 1) / kDecodeSplitTile;
    const int per = (n128 + kDecodeSplits - 1) / kDecodeSplits;       // 128-token tiles per split
    const int sub = kDecodeSplitTile / kTile;
    t0 = min(n_tiles, split * per * sub);
    t1 = min(n_tiles, (split + 1) * per * sub);
  }
  const int n = t1 - t0;
  const int32_t *bt = p.block_table + (size_t)b * p.max_pages;

  // validate the block-table entries this CTA will read
  bool bad_page = false;
  if (n > 0) {
    const int pg0 = t0 * (kTile / kPageSize);
    const int pg1 = (min(L, t1 * kTile) + kPageSize - 1) / kPageSize;
    for (int i = pg0 + tid; i < pg1; i += nthr) {
      const int pg = __ldg(bt + i);
      bad_page |= (pg < 0) | (pg >= p.num_pages);
    }
  }
  const bool any_bad = __syncthreads_or(bad_page) != 0;
  if (tid == 0 && (any_bad || bad_len))
    raise_error(p.err, any_bad ? ATTN_DEVERR_BLOCK_TABLE : ATTN_DEVERR_SEQ_LEN);

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float m_pv = -INFINITY, l_part = 0.f;
  bool failed = false;

  if (!any_bad && n > 0) {
    // q (pre-scaled into the log2 domain) and barriers
    const uint16_t *qg = p.q + ((size_t)b * p.h_q + (size_t)hk * G) * D;
    for (int i = tid; i < G * D; i += nthr) q_s[i] = bf16_to_f32(qg[i]) * p.scale_log2;
    if (tid == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      for (int s = 0; s < kKStages; ++s) mbar_init(&kfull[s], 1);
      for (int s = 0; s < kVStages; ++s) mbar_init(&vfull[s], 1);
      fence_barrier_init();
    }
    __syncthreads();

    // copies of one 32-token tile (K or V): pages of the tile inside [0, L)
    auto issue_tile = [&](const CUtensorMap *map, uint8_t *slot, uint64_t *bar, int tile) {
      const int tok0 = (t0 + tile) * kTile;
      const int npg = (min(L - tok0, kTile) + kPageSize - 1) / kPageSize;   // 1 or 2
      mbar_arrive_expect_tx(bar, npg * Lay::kHalves * Lay::kBoxBytes);
      for (int g = 0; g < npg; ++g) {
        const int page = __ldg(bt + tok0 / kPageSize + g);
        for (int h = 0; h < Lay::kHalves; ++h)
          tma_load_3d(slot + h * 4096 + g * Lay::kBoxBytes, map, bar, h * 64, hk, page * kPageSize);
      }
    };

    int k_issued = 0, v_issued = 0, v_used = 0;
    if (tid == 0) {
      for (; k_issued < min(n, kKStages); ++k_issued)
        issue_tile(&kmap, ks_base + k_issued * Lay::kSlot, &kfull[k_issued], k_issued);
    }

    float m_run = -INFINITY;
    uint32_t kept_bits = 0;
    unsigned long long n_skip = 0;
    const bool skipping = p.thr_log2 > -INFINITY;

    for (int i = 0; i < n + kLookahead; ++i) {
      if (i < n) {
        // ---------------- score pass, tile i ----------------
        const int ks = i % kKStages;
        const bool ok = mbar_wait(&kfull[ks], (i / kKStages) & 1, p.err);
        const uint8_t *kslot = ks_base + ks * Lay::kSlot;
        const int tok = (t0 + i) * kTile + lane;
        float s = -INFINITY;
        if (ok && tok < L) {
          const float *qw = q_s + w * D;
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int h = 0; h < Lay::kHalves; ++h) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 kv = *reinterpret_cast<const uint4 *>(kslot + h * 4096 + sw128_offset(lane, c));
              const float4 qa = *reinterpret_cast<const float4 *>(qw + h * 64 + c * 8);
              const float4 qb = *reinterpret_cast<const float4 *>(qw + h * 64 + c * 8 + 4);
              a0 = fmaf(qa.x, bf16_lo(kv.x), a0); a1 = fmaf(qa.y, bf16_hi(kv.x), a1);
              a0 = fmaf(qa.z, bf16_lo(kv.y), a0); a1 = fmaf(qa.w, bf16_hi(kv.y), a1);
              a0 = fmaf(qb.x, bf16_lo(kv.z), a0); a1 = fmaf(qb.y, bf16_hi(kv.z), a1);
              a0 = fmaf(qb.z, bf16_lo(kv.w), a0); a1 = fmaf(qb.w, bf16_hi(kv.w), a1);
            }
          }
          s = a0 + a1;
        }
        const float tm = warp_max(s);
        // a head votes skip when exp(tile max - running max) < threshold
        const bool vote = (tm == -INFINITY) || (tm - m_run < p.thr_log2);
        m_run = fmaxf(m_run, tm);
        s_ring[(i % kRing) * nthr + tid] = s;
        tm_ring[(i % kRing) * nthr + tid] = tm;
        if (__syncthreads_or(!ok)) { failed = true; break; }
        const bool skip = skipping && (__syncthreads_and(vote) != 0);
        // every thread is done with K slot ks and with the V slot reused below
        if (tid == 0) {
          if (k_issued < n) {
            issue_tile(&kmap, ks_base + ks * Lay::kSlot, &kfull[ks], k_issued);
            ++k_issued;
          }
          if (!skip) {
            const int vs = v_issued % kVStages;
            issue_tile(&vmap, vs_base + vs * Lay::kSlot, &vfull[vs], i);
            ++v_issued;
          } else {
            ++n_skip;
            if (p.skip_mask) {
              const long long unit = ((long long)b * p.h_kv + hk) * p.kt_max + (t0 + i);
              atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
            }
          }
        }
        kept_bits = (kept_bits & ~(1u << (i & 31))) | (uint32_t(!skip) << (i & 31));
      }
      const int j = i - kLookahead;
      if (j >= 0 && ((kept_bits >> (j & 31)) & 1u)) {
        // ---------------- PV pass, tile j ----------------
        const int vs = v_used % kVStages;
        const bool ok = mbar_wait(&vfull[vs], (v_used / kVStages) & 1, p.err);
        ++v_used;
        if (!ok) { failed = true; }
        const float tmj = tm_ring[(j % kRing) * nthr + tid];
        const float sj = s_ring[(j % kRing) * nthr + tid];
        const float m_new = fmaxf(m_pv, tmj);
        const float alpha = ex2(m_pv - m_new);
        l_part *= alpha;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= alpha;
        m_pv = m_new;
        const float pj = ex2(sj - m_new);
        l_part += pj;
        const int nvalid = ok ? min(kTile, L - (t0 + j) * kTile) : 0;
        const uint8_t *vslot = vs_base + vs * Lay::kSlot;
        for (int t = 0; t < nvalid; ++t) {
          const float pt = __shfl_sync(0xffffffffu, pj, t);
          float vv[E];
          pv_load<D>(vslot, t, lane, vv);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = fmaf(pt, vv[e], acc[e]);
        }
      }
    }
    failed = __syncthreads_or(failed) != 0;
    if (failed && tid == 0) {
      // drain copies still in flight before the CTA's shared memory goes away
      for (int x = k_issued - min(kKStages, k_issued); x < k_issued; ++x)
        mbar_wait(&kfull[x % kKStages], (x / kKStages) & 1, nullptr);
      for (int x = v_used; x < v_issued; ++x)
        mbar_wait(&vfull[x % kVStages], (x / kVStages) & 1, nullptr);
    }
    if (tid == 0 && p.skip_counts) {
      atomicAdd(p.skip_counts + 0, (unsigned long long)n);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
  }

  // ---------------- epilogue ----------------
  const float l = warp_sum(l_part);
  const bool dead = any_bad || failed;
  if (p.sequential) {
    const float inv = (l > 0.f && !dead) ? 1.f / l : 0.f;
    uint16_t *o = p.out + ((size_t)b * p.h_q + hq) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = f32_to_bf16(acc[e] * inv);
    if (p.lse && lane == 0)
      p.lse[(size_t)b * p.h_q + hq] = (l > 0.f && !dead) ? (m_pv + __log2f(l)) * kLn2 : -INFINITY;
  } else {
    const size_t row = ((size_t)b * p.h_q + hq) * nsplit + split;
    float *wo = p.ws_o + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) wo[e] = dead ? 0.f : acc[e];
    if (lane == 0) {
      p.ws_ml[row * 2 + 0] = dead ? -INFINITY : m_pv;
      p.ws_ml[row * 2 + 1] = dead ? -1.f : l;      // -1 marks a split that saw bad data
    }
  }
}

// One warp per (sequence, q-head): log-sum-exp combine of the 32 split partials.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeParams p) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= (long long)p.batch * p.h_q) return;
  const float *ml = p.ws_ml + row * kDecodeSplits * 2;
  const float m_s = ml[lane * 2 + 0];
  const float l_s = ml[lane * 2 + 1];
  const bool bad = __any_sync(0xffffffffu, l_s < 0.f);
  const float M = warp_max(m_s);
  const float w_s = (m_s == -INFINITY) ? 0.f : ex2(m_s - M);
  const float Lsum = warp_sum(w_s * l_s);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const float *os = p.ws_o + row * kDecodeSplits * D + lane * E;
  for (int s = 0; s < kDecodeSplits; ++s) {
    const float ws = __shfl_sync(0xffffffffu, w_s, s);
    if (ws == 0.f) continue;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(ws, os[(size_t)s * D + e], acc[e]);
  }
  const bool live = (Lsum > 0.f) && !bad;
  const float inv = live ? 1.f / Lsum : 0.f;
  uint16_t *o = p.out + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] = f32_to_bf16(acc[e] * inv);
  if (p.lse && lane == 0) p.lse[row] = live ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
}

template <int D>
cudaError_t launch_d(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
  const size_t smem = DecodeLayout<D>::bytes(p.group);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.sequential ? 1 : kDecodeSplits, p.h_kv, p.batch);
  decode_kernel<D><<<grid, p.group * 32, smem, stream>>>(kmap, vmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.sequential) return e;
  const long long rows = (long long)p.batch * p.h_q;
  decode_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128>(p, kmap, vmap, stream) : launch_d<64>(p, kmap, vmap, stream);
}

}  // namespace attn
