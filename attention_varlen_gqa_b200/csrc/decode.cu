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
// One CTA (4 warps) = one (sequence b, kv-head hk, split).  The G = h_q / h_kv
// query heads of the group are the 16 rows (zero-padded) of a warp-level bf16
// MMA, so a warp turns 16 tokens x 128 dims of K into the group's scores with
// 16 m16n8k16 MMAs instead of thousands of scalar FMAs; this keeps the kernel
// on the memory side of its roofline.  K and V pages are gathered through the
// block table with 3-D TMA copies (box = 64 dims x 1 head x 16 tokens,
// 128-byte swizzle) into shared-memory rings, 64 tokens (4 pages) per chunk,
// warp w owning tokens [16w, 16w + 16) of every chunk.
// Two passes one chunk apart:
//   score pass (chunk i):  S = Q K^T, per-head maxima of the two 32-token skip
//       tiles of the chunk (exchanged between warps through shared memory),
//       the skip vote of every head against the running max, and the V copy
//       of the pages of the kept tiles only;
//   PV pass (chunk i - 1): per-warp online softmax and O += P V (P taken from
//       the score fragments, V fragments by ldmatrix.trans).
// For thresholds <= 1 a skipped tile never raises the running max, so the
// decisions need only K, and skipped tiles cost no V traffic.  The four
// warps' (m, l, O) are merged at the end.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kChunk = 64;              // tokens per chunk (4 pages)
constexpr int kWarps = 4;               // 16 tokens of each chunk per warp
constexpr int kThreads = 32 * kWarps;
constexpr int kKStages = 3;             // K ring depth (chunks)
constexpr int kLookahead = 1;           // PV pass lags the score pass by this many chunks
constexpr int kVStages = kLookahead + 1;
constexpr int kRing = kLookahead + 1;   // score fragments kept for the PV pass
static_assert(kDecodeSplits == 32, "the combine kernel gives one lane per split");
static_assert(kDecodeSplitTile % kChunk == 0, "a split is a whole number of chunks");
static_assert(kChunk == 2 * kSkipTile, "a chunk holds two skip tiles");

template <int D>
struct DecodeLayout {
  static constexpr int kSlot = kChunk * D * 2;        // bytes of one K or V chunk
  static constexpr int kHalfBytes = kChunk * 128;     // one 64-dim half: 64 rows x 128 B
  static constexpr int kBoxBytes = 16 * 64 * 2;       // one TMA box: 16 tokens x 64 dims
  static constexpr int kHalves = D / 64;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKStages * kSlot;
  static constexpr int kS = kV + kVStages * kSlot;                 // [ring][warp][lane][8] fp32
  static constexpr int kQmax = kS + kRing * kWarps * 32 * 8 * 4;   // [2][warp][16] fp32
  static constexpr int kBar = kQmax + 2 * kWarps * 16 * 4;
  static constexpr int kEnd = kBar + (kKStages + kVStages) * 8;
  // the end-of-CTA merge reuses the K ring: [warp][16] m, [warp][16] l, [warp][16][D] O
  static constexpr int kMerge = kWarps * 16 * 4 * 2 + kWarps * 16 * D * 4;
  static_assert(kMerge <= kKStages * kSlot, "merge area fits the K ring");
  static constexpr size_t kBytes = 1024 + kEnd;
};

ATTN_DEVICE uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Address of the 16-byte chunk holding dims [8c, 8c + 8) of token `tok` inside
// a swizzled chunk slot (64-dim halves of 64 rows x 128 B).
template <int D>
ATTN_DEVICE uint32_t slot_addr(uint32_t slot, int tok, int c8) {
  return slot + (c8 >> 3) * DecodeLayout<D>::kHalfBytes + tok * 128 + (((c8 & 7) ^ (tok & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap,
                                                          DecodeParams p) {
  using Lay = DecodeLayout<D>;
  constexpr int KS = D / 16;                          // k-steps of the score MMA
  constexpr int NT = D / 8;                           // n-tiles of the PV MMA
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const uint32_t sK = smem_u32(base + Lay::kK);
  const uint32_t sV = smem_u32(base + Lay::kV);
  float *s_ring = reinterpret_cast<float *>(base + Lay::kS);
  float *qmax = reinterpret_cast<float *>(base + Lay::kQmax);
  uint64_t *kfull = reinterpret_cast<uint64_t *>(base + Lay::kBar);
  uint64_t *vfull = kfull + kKStages;

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.group;
  const int nsplit = gridDim.x;
  const int r0 = lane >> 2, r1 = r0 + 8;              // MMA rows (query heads) of this lane
  const int cq = (lane & 3) * 2;                      // first column of this lane in a fragment

  int L = __ldg(p.seq_lens + b);
  const bool bad_len = (L < 0) | (L > p.max_pages * kPageSize);
  if (bad_len) L = 0;
  const int n_chunks_all = (L + kChunk - 1) / kChunk;
  int c0 = 0, c1 = n_chunks_all;
  if (!p.sequential) {
    const int n128 = (L + kDecodeSplitTile - 1) / kDecodeSplitTile;
    const int per = (n128 + kDecodeSplits - 1) / kDecodeSplits;   // 128-token tiles per split
    const int sub = kDecodeSplitTile / kChunk;
    c0 = min(n_chunks_all, split * per * sub);
    c1 = min(n_chunks_all, (split + 1) * per * sub);
  }
  const int n = c1 - c0;
  const int32_t *bt = p.block_table + (size_t)b * p.max_pages;

  // validate the block-table entries this CTA will read
  bool bad_page = false;
  if (n > 0) {
    const int pg0 = c0 * (kChunk / kPageSize);
    const int pg1 = (min(L, c1 * kChunk) + kPageSize - 1) / kPageSize;
    for (int i = pg0 + tid; i < pg1; i += kThreads) {
      const int pg = __ldg(bt + i);
      bad_page |= (pg < 0) | (pg >= p.num_pages);
    }
  }
  const bool any_bad = __syncthreads_or(bad_page) != 0;
  if (tid == 0 && (any_bad || bad_len))
    raise_error(p.err, any_bad ? ATTN_DEVERR_BLOCK_TABLE : ATTN_DEVERR_SEQ_LEN);

  float o_acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) o_acc[t][e] = 0.f;
  float m_w[2] = {-INFINITY, -INFINITY};              // this warp's running max, rows r0 / r1
  float l_w[2] = {0.f, 0.f};                          // partial row sums (this lane's columns)
  bool failed = false;

  if (!any_bad && n > 0) {
    if (tid == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      for (int s = 0; s < kKStages; ++s) mbar_init(&kfull[s], 1);
      for (int s = 0; s < kVStages; ++s) mbar_init(&vfull[s], 1);
      fence_barrier_init();
    }
    // query fragments (A operand, rows = heads of the group, zero beyond G)
    uint32_t qa[KS][4];
    {
      const uint16_t *qg = p.q + ((size_t)b * p.h_q + (size_t)hk * G) * D;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int d0 = kk * 16 + cq;
        qa[kk][0] = r0 < G ? *reinterpret_cast<const uint32_t *>(qg + (size_t)r0 * D + d0) : 0u;
        qa[kk][1] = r1 < G ? *reinterpret_cast<const uint32_t *>(qg + (size_t)r1 * D + d0) : 0u;
        qa[kk][2] = r0 < G ? *reinterpret_cast<const uint32_t *>(qg + (size_t)r0 * D + d0 + 8) : 0u;
        qa[kk][3] = r1 < G ? *reinterpret_cast<const uint32_t *>(qg + (size_t)r1 * D + d0 + 8) : 0u;
      }
    }
    __syncthreads();

    // copies of the pages [pg_lo, pg_hi) of chunk c (relative index) into a slot
    auto issue_pages = [&](const CUtensorMap *map, uint32_t slot, uint64_t *bar, int c, int pg_lo,
                           int pg_hi) {
      const int tok0 = (c0 + c) * kChunk;
      const int npg = (min(L - tok0, kChunk) + kPageSize - 1) / kPageSize;     // pages inside [0, L)
      pg_hi = min(pg_hi, npg);
      const int cnt = max(0, pg_hi - pg_lo);
      mbar_arrive_expect_tx(bar, cnt * Lay::kHalves * Lay::kBoxBytes);
      for (int g = pg_lo; g < pg_hi; ++g) {
        const int page = __ldg(bt + tok0 / kPageSize + g);
        for (int h = 0; h < Lay::kHalves; ++h)
          tma_load_3d(base + (slot - smem_u32(base)) + h * Lay::kHalfBytes + g * Lay::kBoxBytes, map, bar,
                      h * 64, hk, page * kPageSize);
      }
    };

    int k_issued = 0, v_issued = 0, v_used = 0;
    if (tid == 0)
      for (; k_issued < min(n, kKStages); ++k_issued)
        issue_pages(&kmap, sK + k_issued * Lay::kSlot, &kfull[k_issued], k_issued, 0, 4);

    float m_run[kMaxGroup];                           // running max per head (log2 units)
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) m_run[h] = -INFINITY;
    uint32_t kept_bits = 0;                           // 2 bits per chunk: tiles A, B kept
    unsigned long long n_vis = 0, n_skip = 0;
    const bool skipping = p.thr_log2 > -INFINITY;
    const float sl2 = p.scale_log2;

    for (int i = 0; i < n + kLookahead; ++i) {
      if (i < n) {
        // ---------------- score pass, chunk i ----------------
        const int ks = i % kKStages;
        const bool ok = mbar_wait(&kfull[ks], (i / kKStages) & 1, p.err) && !failed;
        const uint32_t kslot = sK + ks * Lay::kSlot;
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
        if (ok) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int tok = w * 16 + nt * 8 + (lane & 7);
#pragma unroll
            for (int m = 0; m < D / 32; ++m) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4(slot_addr<D>(kslot, tok, m * 4 + (lane >> 3)), b0, b1, b2, b3);
              mma_bf16_16816(sc[nt], qa[2 * m], b0, b1);
              mma_bf16_16816(sc[nt], qa[2 * m + 1], b2, b3);
            }
          }
        }
        // scale into the log2 domain, mask tokens beyond L and padding rows
        const int tok_base = (c0 + i) * kChunk + w * 16;
        float qm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tok_base + nt * 8 + cq + (e & 1);
            const int row = (e < 2) ? r0 : r1;
            const float v = (tok < L && row < G) ? sc[nt][e] * sl2 : -INFINITY;
            sc[nt][e] = v;
            qm[e >> 1] = fmaxf(qm[e >> 1], v);
          }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          qm[h] = fmaxf(qm[h], __shfl_xor_sync(0xffffffffu, qm[h], 1));
          qm[h] = fmaxf(qm[h], __shfl_xor_sync(0xffffffffu, qm[h], 2));
        }
        float *qx = qmax + ((i & 1) * kWarps + w) * 16;
        if ((lane & 3) == 0) {
          qx[r0] = qm[0];
          qx[r1] = qm[1];
        }
        float *sr = s_ring + (((i % kRing) * kWarps + w) * 32 + lane) * 8;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sr[nt * 4 + e] = sc[nt][e];
        if (__syncthreads_or(!ok)) {
          failed = true;
          break;
        }
        // every warp is done with K slot ks; the per-head maxima are visible
        const float *qa_x = qmax + (i & 1) * kWarps * 16;
        bool keep[2] = {true, true};
        const bool vis_b = (c0 + i) * kChunk + kSkipTile < L;
        if (skipping) {
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            bool all = true;
            for (int h = 0; h < G; ++h) {
              const float tm = fmaxf(qa_x[(2 * tt) * 16 + h], qa_x[(2 * tt + 1) * 16 + h]);
              // a head votes skip when exp(tile max - running max) < threshold
              all = all && ((tm == -INFINITY) || (tm - m_run[h] < p.thr_log2));
              m_run[h] = fmaxf(m_run[h], tm);
            }
            keep[tt] = !all;
          }
        }
        if (!vis_b) keep[1] = false;
        if (tid == 0) {
          if (k_issued < n) {
            issue_pages(&kmap, sK + ks * Lay::kSlot, &kfull[ks], k_issued, 0, 4);
            ++k_issued;
          }
          if (keep[0] || keep[1]) {
            const int vs = v_issued % kVStages;
            // pages 0-1 hold tile A, pages 2-3 tile B
            if (keep[0] && keep[1])
              issue_pages(&vmap, sV + vs * Lay::kSlot, &vfull[vs], i, 0, 4);
            else if (keep[0])
              issue_pages(&vmap, sV + vs * Lay::kSlot, &vfull[vs], i, 0, 2);
            else
              issue_pages(&vmap, sV + vs * Lay::kSlot, &vfull[vs], i, 2, 4);
            ++v_issued;
          }
          n_vis += 1 + (vis_b ? 1 : 0);
          for (int tt = 0; tt < 2; ++tt) {
            if (tt == 1 && !vis_b) break;
            if (!keep[tt]) {
              ++n_skip;
              if (p.skip_mask) {
                const long long unit = ((long long)b * p.h_kv + hk) * p.kt_max + 2 * (c0 + i) + tt;
                atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
              }
            }
          }
        }
        const uint32_t kb = (keep[0] ? 1u : 0u) | (keep[1] ? 2u : 0u);
        kept_bits = (kept_bits & ~(3u << (2 * (i & 15)))) | (kb << (2 * (i & 15)));
      }
      const int j = i - kLookahead;
      if (j >= 0) {
        const uint32_t kb = (kept_bits >> (2 * (j & 15))) & 3u;
        if (kb != 0u) {
          // ---------------- PV pass, chunk j ----------------
          const int vs = v_used % kVStages;
          const bool okv = mbar_wait(&vfull[vs], (v_used / kVStages) & 1, p.err);
          ++v_used;
          if (!okv) failed = true;
          const bool mine = ((kb >> (w >> 1)) & 1u) != 0u;   // warps 0-1: tile A, 2-3: tile B
          if (okv && mine) {
            const uint32_t vslot = sV + vs * Lay::kSlot;
            const int tok_base = (c0 + j) * kChunk + w * 16;
            // V rows of tokens at or beyond L are not data of this sequence: zero them
            if (tok_base + 16 > L) {
              for (int x = lane; x < 16 * (D / 8); x += 32) {
                const int t = x / (D / 8), c8 = x % (D / 8);
                if (tok_base + t >= L) {
                  uint8_t *pz = base + (slot_addr<D>(vslot, w * 16 + t, c8) - smem_u32(base));
                  *reinterpret_cast<uint4 *>(pz) = make_uint4(0u, 0u, 0u, 0u);
                }
              }
              fence_proxy_async_smem();   // a later TMA copy reuses this slot
              __syncwarp();
            }
            const float *sr = s_ring + (((j % kRing) * kWarps + w) * 32 + lane) * 8;
            float s[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) s[nt][e] = sr[nt * 4 + e];
            // online softmax of this warp's rows over its 16 tokens
            float mx[2];
            mx[0] = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
            mx[1] = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
              mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
              const float m_new = fmaxf(m_w[h], mx[h]);
              alpha[h] = (m_w[h] == -INFINITY) ? 0.f : ex2(m_w[h] - m_new);
              m_w[h] = m_new;
              l_w[h] *= alpha[h];
            }
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                o_acc[t][0] *= alpha[0];
                o_acc[t][1] *= alpha[0];
                o_acc[t][2] *= alpha[1];
                o_acc[t][3] *= alpha[1];
              }
            }
            const float mr0 = (m_w[0] == -INFINITY) ? 0.f : m_w[0];
            const float mr1 = (m_w[1] == -INFINITY) ? 0.f : m_w[1];
            uint32_t pa[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const float p0 = ex2(s[nt][0] - mr0), p1 = ex2(s[nt][1] - mr0);
              const float p2 = ex2(s[nt][2] - mr1), p3 = ex2(s[nt][3] - mr1);
              l_w[0] += p0 + p1;
              l_w[1] += p2 + p3;
              pa[2 * nt + 0] = pack_bf16x2(p0, p1);
              pa[2 * nt + 1] = pack_bf16x2(p2, p3);
            }
            // A fragment order: (rows r0, tokens 0-7), (rows r1, 0-7), (r0, 8-15), (r1, 8-15)
            const uint32_t afr[4] = {pa[0], pa[1], pa[2], pa[3]};
#pragma unroll
            for (int q2 = 0; q2 < NT / 2; ++q2) {
              // matrices: (tokens 0-7, dims 16q2..+7), (tokens 8-15, same), (0-7, +8..+15), (8-15, +8..+15)
              const int mtx = lane >> 3;
              const int tok = w * 16 + (mtx & 1) * 8 + (lane & 7);
              const int c8 = 2 * q2 + (mtx >> 1);
              uint32_t b0, b1, b2, b3;
              ldsm_x4_trans(slot_addr<D>(vslot, tok, c8), b0, b1, b2, b3);
              mma_bf16_16816(o_acc[2 * q2], afr, b0, b1);
              mma_bf16_16816(o_acc[2 * q2 + 1], afr, b2, b3);
            }
          }
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
      atomicAdd(p.skip_counts + 0, n_vis);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
    __syncthreads();
  }

  // ---------------- merge the four warps ----------------
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_w[h] += __shfl_xor_sync(0xffffffffu, l_w[h], 1);
    l_w[h] += __shfl_xor_sync(0xffffffffu, l_w[h], 2);
  }
  float *mm = reinterpret_cast<float *>(base + Lay::kK);        // [warp][16]
  float *ll = mm + kWarps * 16;                                  // [warp][16]
  float *oo = ll + kWarps * 16;                                  // [warp][16][D]
  if ((lane & 3) == 0) {
    mm[w * 16 + r0] = m_w[0];
    mm[w * 16 + r1] = m_w[1];
    ll[w * 16 + r0] = l_w[0];
    ll[w * 16 + r1] = l_w[1];
  }
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    *reinterpret_cast<float2 *>(oo + ((size_t)w * 16 + r0) * D + t * 8 + cq) = make_float2(o_acc[t][0], o_acc[t][1]);
    *reinterpret_cast<float2 *>(oo + ((size_t)w * 16 + r1) * D + t * 8 + cq) = make_float2(o_acc[t][2], o_acc[t][3]);
  }
  __syncthreads();
  const bool dead = any_bad || failed;
  for (int x = tid; x < G * D; x += kThreads) {
    const int h = x / D, d = x % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, mm[ww * 16 + h]);
    float Lsum = 0.f, acc = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kWarps; ++ww) {
        const float mw = mm[ww * 16 + h];
        const float sc = (mw == -INFINITY) ? 0.f : ex2(mw - M);
        Lsum += sc * ll[ww * 16 + h];
        acc += sc * oo[((size_t)ww * 16 + h) * D + d];
      }
    }
    const int hq = hk * G + h;
    if (p.sequential) {
      const bool live = Lsum > 0.f && !dead;
      p.out[((size_t)b * p.h_q + hq) * D + d] = f32_to_bf16(live ? acc / Lsum : 0.f);
      if (d == 0 && p.lse)
        p.lse[(size_t)b * p.h_q + hq] = live ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
    } else {
      const size_t row = ((size_t)b * p.h_q + hq) * nsplit + split;
      p.ws_o[row * D + d] = dead ? 0.f : acc;
      if (d == 0) {
        p.ws_ml[row * 2 + 0] = dead ? -INFINITY : M;
        p.ws_ml[row * 2 + 1] = dead ? -1.f : Lsum;   // -1 marks a split that saw bad data
      }
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
  const size_t smem = DecodeLayout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.sequential ? 1 : kDecodeSplits, p.h_kv, p.batch);
  decode_kernel<D><<<grid, kThreads, smem, stream>>>(kmap, vmap, p);
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
