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
// One CTA (4 warps) = one (sequence b, kv-head hk, split).  A warp turns 16
// tokens x 128 dims of K into the group's scores with warp-level bf16 MMAs,
// computed transposed (S^T = K Q^T, O^T = V^T P^T): the 16 tokens are the MMA
// rows and the G = h_q / h_kv query heads of the group its columns, in tiles
// of 8 (zero-padded), so a group of up to 8 heads costs 8 m16n8k16 MMAs per 16
// tokens for the scores and 8 for P V.  K and V pages are gathered through the
// block table with 3-D TMA copies (box = 64 dims x 1 head x 16 tokens,
// 128-byte swizzle) into shared memory, 64 tokens (4 pages) per chunk, warp w
// owning tokens [16w, 16w + 16) of every chunk.  Each warp keeps its own
// online-softmax state (m, l, O) over its tokens; the four are merged at the
// end of the CTA.
//
// Dense schedule: K and V of a chunk travel together through a 2-stage ring
// and every chunk is finished (S, softmax, PV) in the iteration it arrives.
// Sequential skip schedule: two passes two chunks apart over a ring of chunk
// slots, where a slot first receives a chunk's K and, once the score pass is
// done with it, the V pages of that chunk's kept tiles --
//   score pass (chunk i):  S = Q K^T, per-head maxima of the chunk's two
//       32-token skip tiles (exchanged between warps through shared memory),
//       the skip vote of every head against the running max, and the V copy
//       of the kept tiles' pages only;
//   PV pass (chunk i - 2): online softmax and O += P V of the kept tiles, after
//       which the slot takes the K of chunk i - 2 + kSeqSlots.
// For thresholds <= 1 a skipped tile never raises the running max, so the
// decisions need only K, and skipped tiles cost no V traffic.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4.cuh"

namespace attn {
namespace {

constexpr int kChunk = 64;              // tokens per chunk (4 pages)
constexpr int kWarps = 4;               // 16 tokens of each chunk per warp
constexpr int kThreads = 32 * kWarps;
// dense: K+V chunks in the ring.  Two stages (66 KB) let three CTAs share an
// SM: more warps to cover the per-chunk latencies than two CTAs with three
// stages each, for the same bytes in flight (measured 0.736 vs 0.820 ms).
constexpr int kDenseStages = 2;
constexpr int kSeqSlots = 5;            // sequential: chunk slots; a slot holds a chunk's K, then its V
constexpr int kSeqLookahead = 2;        // sequential: PV pass lags the score pass
constexpr int kSeqRing = kSeqLookahead + 1;
constexpr int kRingFloats = 12;         // sequential: a lane's 8 scores + 4 head maxima per chunk
static_assert(kSeqSlots > kSeqLookahead + 1, "K prefetch depth is kSeqSlots - kSeqLookahead");
static_assert(kDecodeSplits == 32, "the combine kernel gives one lane per split");
static_assert(kDecodeSplitTile % kChunk == 0, "a split is a whole number of chunks");
static_assert(kChunk == 2 * kSkipTile, "a chunk holds two skip tiles");

template <int D, bool SEQ>
struct DecodeLayout {
  static constexpr int kSlot = kChunk * D * 2;        // bytes of one K or V chunk
  // dense: stage s holds K at 2s * kSlot and V at (2s + 1) * kSlot
  static constexpr int kK = 0;
  static constexpr int kS = SEQ ? kSeqSlots * kSlot : 2 * kDenseStages * kSlot;
  static constexpr int kQmax = kS + (SEQ ? kSeqRing * kWarps * 32 * kRingFloats * 4 : 0);
  // sequential: the walk's running max after each tile, [ring][tile][head] (QDQ)
  static constexpr int kMrun = kQmax + (SEQ ? 2 * kWarps * 16 * 4 : 0);
  static constexpr int kBar = kMrun + (SEQ ? kSeqRing * 2 * kMaxGroup * 4 : 0);
  static constexpr int kNumBars = SEQ ? 2 * kSeqSlots : kDenseStages;
  static constexpr int kBt = kBar + kNumBars * 8;                  // the CTA's block-table entries
  static constexpr int kBtCap = SEQ ? 2048 : 256;                  // entries (longer ranges read global)
  static constexpr int kEnd = kBt + kBtCap * 4;
  // the end-of-CTA merge reuses the K / V slots (no copy is in flight by then):
  // [warp][16] m, [warp][16] l, [warp][16][D] O
  static constexpr int kMerge = kWarps * 16 * 4 * 2 + kWarps * 16 * D * 4;
  static_assert(kMerge <= (SEQ ? kSeqSlots : 2 * kDenseStages) * kSlot, "merge area fits");
  static constexpr size_t kBytes = 1024 + kEnd;
};

ATTN_DEVICE uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Address of the 16-byte chunk holding dims [8c, 8c + 8) of token `tok` inside
// a swizzled chunk slot (64-dim halves of 64 rows x 128 B).
ATTN_DEVICE uint32_t slot_addr(uint32_t slot, int tok, int c8) {
  return slot + (c8 >> 3) * (kChunk * 128) + tok * 128 + (((c8 & 7) ^ (tok & 7)) << 4);
}

// Per-lane geometry of the m16n8k16 fragments: g = the lane's row of an 8-row
// fragment, cq = its first column of a column pair.
struct Lane {
  int w, lane, g, cq;
  ATTN_DEVICE explicit Lane(int tid)
      : w(tid >> 5), lane(tid & 31), g((tid & 31) >> 2), cq(((tid & 31) & 3) * 2) {}
};

// Query fragments as the B operand of S^T = K Q^T: qb[n][kk] = the two 8-dim
// halves of dims [16 kk, 16 kk + 16) of head 8 n + g (zero beyond G).
template <int D, int NH>
ATTN_DEVICE void load_q_frags(uint32_t (&qb)[NH][D / 16][2], const uint16_t *qg, int G, const Lane &ln) {
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    const int h = 8 * n + ln.g;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint16_t *src = qg + (size_t)h * D + kk * 16 + ln.cq;
      qb[n][kk][0] = h < G ? *reinterpret_cast<const uint32_t *>(src) : 0u;
      qb[n][kk][1] = h < G ? *reinterpret_cast<const uint32_t *>(src + 8) : 0u;
    }
  }
}

// Scores of this warp's 16 tokens, computed transposed (M = the 16 tokens,
// N = the group's heads in tiles of 8, K = head dims) so that a group of G <= 8
// heads pads to 8 MMA columns, not 16 rows: sc[n][e] = S(head 8 n + cq + (e & 1),
// token tok_base + g + 8 (e >> 1)) in the log2 domain, -inf for tokens at or
// beyond L and for padding heads; qm[n][h] = max over the 16 tokens of head
// 8 n + cq + h.
template <int D, int NH>
ATTN_DEVICE void warp_scores(float (&sc)[NH][4], float (&qm)[NH][2], uint32_t kslot,
                             const uint32_t (&qb)[NH][D / 16][2], int tok_base, int L, int G, float sl2,
                             const Lane &ln) {
  // even and odd k-steps accumulate separately: two chains of D / 32 MMAs
  float acc[NH][2][4];
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][0][e] = acc[n][1][e] = 0.f;
  // A fragments (K rows): matrices (tokens 0-7, dims 0-7), (8-15, 0-7), (0-7, 8-15), (8-15, 8-15)
  const int tok = ln.w * 16 + (ln.lane & 7) + ((ln.lane >> 3) & 1) * 8;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(slot_addr(kslot, tok, 2 * kk + (ln.lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n = 0; n < NH; ++n) mma_bf16_16816(acc[n][kk & 1], a, qb[n][kk][0], qb[n][kk][1]);
  }
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    qm[n][0] = qm[n][1] = -INFINITY;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = tok_base + ln.g + 8 * (e >> 1);
      const int h = 8 * n + ln.cq + (e & 1);
      const float v = (t < L && h < G) ? (acc[n][0][e] + acc[n][1][e]) * sl2 : -INFINITY;
      sc[n][e] = v;
      qm[n][e & 1] = fmaxf(qm[n][e & 1], v);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) qm[n][h] = fmaxf(qm[n][h], __shfl_xor_sync(0xffffffffu, qm[n][h], o));
  }
}

// V rows of tokens at or beyond L are not data of this sequence: zero this
// warp's ones before they meet a zero probability inside the MMA.
template <int D>
ATTN_DEVICE void zero_tail_rows(uint8_t *base, uint32_t vslot, int tok_base, int L, const Lane &ln) {
  if (tok_base + 16 <= L) return;
  for (int x = ln.lane; x < 16 * (D / 8); x += 32) {
    const int t = x / (D / 8), c8 = x % (D / 8);
    if (tok_base + t >= L) {
      uint8_t *pz = base + (slot_addr(vslot, ln.w * 16 + t, c8) - smem_u32(base));
      *reinterpret_cast<uint4 *>(pz) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  fence_proxy_async_smem();   // a later TMA copy reuses this slot
  __syncwarp();
}

// Online-softmax update of this warp's heads with its 16 tokens and
// O^T += V^T P^T (M = head dims, N = heads, K = the 16 tokens).  The lane's
// probabilities come out of the score fragment as (token g, heads cq, cq + 1)
// pairs; one 8x8 register transpose per 8 tokens turns them into the B
// fragment, which wants (tokens cq, cq + 1, head g).  o_acc[mt][n][e] = O(head
// 8 n + cq + (e & 1), dim 16 mt + g + 8 (e >> 1)).
template <int D, int NH>
ATTN_DEVICE void warp_pv(float (&o_acc)[D / 16][NH][4], float (&m_w)[NH][2], float (&l_w)[NH][2],
                         const float (&s)[NH][4], const float (&qm)[NH][2], uint32_t vslot, const Lane &ln) {
  float alpha[NH][2];
  bool rescale = false;
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float m_new = fmaxf(m_w[n][h], qm[n][h]);
      alpha[n][h] = (m_w[n][h] == -INFINITY) ? 0.f : ex2(m_w[n][h] - m_new);
      m_w[n][h] = m_new;
      l_w[n][h] *= alpha[n][h];
      rescale |= alpha[n][h] != 1.f;
    }
  if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int n = 0; n < NH; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[t][n][e] *= alpha[n][e & 1];
  }
  uint32_t pb[NH][2];
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    const float mr0 = (m_w[n][0] == -INFINITY) ? 0.f : m_w[n][0];
    const float mr1 = (m_w[n][1] == -INFINITY) ? 0.f : m_w[n][1];
    const float p0 = ex2(s[n][0] - mr0), p1 = ex2(s[n][1] - mr1);   // token g
    const float p2 = ex2(s[n][2] - mr0), p3 = ex2(s[n][3] - mr1);   // token g + 8
    l_w[n][0] += p0 + p2;
    l_w[n][1] += p1 + p3;
    pb[n][0] = movmatrix_trans(pack_bf16x2(p0, p1));
    pb[n][1] = movmatrix_trans(pack_bf16x2(p2, p3));
  }
  // A fragments (V^T) by transposing loads: matrices (tokens 0-7, dims 0-7),
  // (0-7, 8-15), (8-15, 0-7), (8-15, 8-15) of the m-tile
  const int tok = ln.w * 16 + (ln.lane & 7) + ((ln.lane >> 4) & 1) * 8;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    uint32_t a[4];
    ldsm_x4_trans(slot_addr(vslot, tok, 2 * mt + ((ln.lane >> 3) & 1)), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int n = 0; n < NH; ++n) mma_bf16_16816(o_acc[mt][n], a, pb[n][0], pb[n][1]);
  }
}

// The lane's entry of a QDQ ratio table (lane j holds entry j & 7).
ATTN_DEVICE float table_entry(const float (&tab)[8], int lane) {
  float t = tab[0];
#pragma unroll
  for (int j = 1; j < 8; ++j)
    if ((lane & 7) == j) t = tab[j];
  return t;
}

// warp_pv with NVFP4 quantise-dequantise of P and / or V.  Every warp takes
// as its reference max the running max of the 32-key walk after this tile,
// mt[n][h] (heads 8 n + cq + h; the same for every warp), so that p =
// exp(s - M_t) as the walk defines it; l sums the unquantised p.  A warp's 16
// tokens are one page, so a P block is one head's 16 p of this warp (8 lanes
// x 2) and a V block one channel's 16 values (4 lanes x 4).  With V quantised
// the P V MMAs take f16 operands (the dequantised products q * s are exact in
// f16), else bf16; O accumulates in units of g_p g_v (p.qdq_out undoes it).
template <int D, int NH>
ATTN_DEVICE void warp_pv_qdq(float (&o_acc)[D / 16][NH][4], float (&m_w)[NH][2], float (&l_w)[NH][2],
                             const float (&s)[NH][4], const float (&mt)[NH][2], uint32_t vslot, const Lane &ln,
                             const DecodeParams &p, float p_tab, float v_tab) {
  float alpha[NH][2];
  bool rescale = false;
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float m_new = fmaxf(m_w[n][h], mt[n][h]);
      alpha[n][h] = (m_w[n][h] == -INFINITY) ? 0.f : ex2(m_w[n][h] - m_new);
      m_w[n][h] = m_new;
      l_w[n][h] *= alpha[n][h];
      rescale |= alpha[n][h] != 1.f;
    }
  if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int n = 0; n < NH; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[t][n][e] *= alpha[n][e & 1];
  }
  const bool vq = p.v_qdq != 0;
  uint32_t pb[NH][2];
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    const float mr0 = (m_w[n][0] == -INFINITY) ? 0.f : m_w[n][0];
    const float mr1 = (m_w[n][1] == -INFINITY) ? 0.f : m_w[n][1];
    const float p0 = ex2(s[n][0] - mr0), p1 = ex2(s[n][1] - mr1);   // token g, heads cq, cq + 1
    const float p2 = ex2(s[n][2] - mr0), p3 = ex2(s[n][3] - mr1);   // token g + 8
    l_w[n][0] += p0 + p2;
    l_w[n][1] += p1 + p3;
    uint32_t x01, x23;                                               // f16x2 operand pairs
    if (p.p_qdq) {
      // block max of heads cq, cq + 1 over the warp's 16 tokens (lanes g = 0..7)
      float b0 = fmaxf(p0, p2), b1 = fmaxf(p1, p3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        b0 = fmaxf(b0, __shfl_xor_sync(0xffffffffu, b0, o));
        b1 = fmaxf(b1, __shfl_xor_sync(0xffffffffu, b1, o));
      }
      const uint32_t sc = e4m3x2_as_f16x2(__fmul_rn(b0, p.p_k), __fmul_rn(b1, p.p_k));
      const float r0 = ratio_from_table(f16_lo(sc), p_tab), r1 = ratio_from_table(f16_hi(sc), p_tab);
      x01 = hmul2_u32(e2m1x2_as_f16x2(__fmul_rn(p0, r0), __fmul_rn(p1, r1)), sc);
      x23 = hmul2_u32(e2m1x2_as_f16x2(__fmul_rn(p2, r0), __fmul_rn(p3, r1)), sc);
      if (!vq) {
        x01 = f16x2_to_bf16x2(x01);
        x23 = f16x2_to_bf16x2(x23);
      }
    } else if (vq) {
      x01 = pack_f16x2(p0, p1);
      x23 = pack_f16x2(p2, p3);
    } else {
      x01 = pack_bf16x2(p0, p1);
      x23 = pack_bf16x2(p2, p3);
    }
    pb[n][0] = movmatrix_trans(x01);
    pb[n][1] = movmatrix_trans(x23);
  }
  const int tok = ln.w * 16 + (ln.lane & 7) + ((ln.lane >> 4) & 1) * 8;
#pragma unroll
  for (int mt_ = 0; mt_ < D / 16; ++mt_) {
    uint32_t a[4];
    ldsm_x4_trans(slot_addr(vslot, tok, 2 * mt_ + ((ln.lane >> 3) & 1)), a[0], a[1], a[2], a[3]);
    if (vq) {
      // a[0], a[2]: channel g of the m-tile, tokens 2 (lane % 4) + {0, 1} and
      // + 8; a[1], a[3]: channel g + 8.  Block max over the 4 lanes of a row.
      uint32_t bm = absmax_pairs_bf16(a[0], a[2], a[1], a[3]);
      bm = max_bf16x2(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
      bm = max_bf16x2(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
      const uint32_t sc = e4m3x2_as_f16x2(__fmul_rn(bf16_lo(bm), p.v_k), __fmul_rn(bf16_hi(bm), p.v_k));
      const float r_g = ratio_from_table(f16_lo(sc), v_tab), r_g8 = ratio_from_table(f16_hi(sc), v_tab);
      const uint32_t s_g = f16x2_bcast(sc, false), s_g8 = f16x2_bcast(sc, true);
      const uint64_t r2_g = f2_pack(r_g, r_g), r2_g8 = f2_pack(r_g8, r_g8);
      uint32_t f[4];
      f[0] = qdq_bf16_pair(a[0], r2_g, s_g);
      f[1] = qdq_bf16_pair(a[1], r2_g8, s_g8);
      f[2] = qdq_bf16_pair(a[2], r2_g, s_g);
      f[3] = qdq_bf16_pair(a[3], r2_g8, s_g8);
#pragma unroll
      for (int n = 0; n < NH; ++n) mma_f16_16816(o_acc[mt_][n], f, pb[n][0], pb[n][1]);
    } else {
#pragma unroll
      for (int n = 0; n < NH; ++n) mma_bf16_16816(o_acc[mt_][n], a, pb[n][0], pb[n][1]);
    }
  }
}

// Merge the four warps' (m, l, O) and write the CTA's result: the split
// partial (dense) or the normalised output and LSE (sequential).
template <int D, int NH>
ATTN_DEVICE void merge_and_store(uint8_t *merge_area, const float (&o_acc)[D / 16][NH][4],
                                 const float (&m_w)[NH][2], float (&l_w)[NH][2], bool dead, int G, int b,
                                 int hk, int split, int nsplit, bool sequential, const DecodeParams &p,
                                 const Lane &ln) {
#pragma unroll
  for (int n = 0; n < NH; ++n)
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) l_w[n][h] += __shfl_xor_sync(0xffffffffu, l_w[n][h], o);
  float *mm = reinterpret_cast<float *>(merge_area);   // [warp][16]
  float *ll = mm + kWarps * 16;                         // [warp][16]
  float *oo = ll + kWarps * 16;                         // [warp][16][D]
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    const int h = 8 * n + ln.cq;
    if (ln.g == 0) {
      mm[ln.w * 16 + h] = m_w[n][0];
      mm[ln.w * 16 + h + 1] = m_w[n][1];
      ll[ln.w * 16 + h] = l_w[n][0];
      ll[ln.w * 16 + h + 1] = l_w[n][1];
    }
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        oo[((size_t)ln.w * 16 + h + (e & 1)) * D + t * 16 + ln.g + 8 * (e >> 1)] = o_acc[t][n][e];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += kThreads) {
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
    if (sequential) {
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

// TMA copies of pages [pg_lo, pg_hi) of the chunk starting at token tok0
// (clipped to the pages inside [0, L)); one expect-tx arrive on `bar`.
// `pages` is indexed by the sequence's page number; it points at the CTA's
// shared-memory copy of its block-table range (or at the global table).
template <int D>
ATTN_DEVICE void issue_pages(const CUtensorMap *map, uint8_t *slot, uint64_t *bar, const int32_t *pages,
                             int tok0, int L, int hk, int pg_lo, int pg_hi, bool arrive) {
  const int npg = (min(L - tok0, kChunk) + kPageSize - 1) / kPageSize;
  pg_hi = min(pg_hi, npg);
  const int cnt = max(0, pg_hi - pg_lo);
  if (arrive) mbar_arrive_expect_tx(bar, cnt * (D / 64) * (16 * 64 * 2));
  for (int g = pg_lo; g < pg_hi; ++g) {
    const int page = pages[tok0 / kPageSize + g];
    for (int h = 0; h < D / 64; ++h)
      tma_load_3d(slot + h * (kChunk * 128) + g * (16 * 64 * 2), map, bar, h * 64, hk, page * kPageSize);
  }
}

template <int D, bool SEQ, int NH, bool QDQ>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap,
                                                          DecodeParams p) {
  static_assert(SEQ || !QDQ, "quantise-dequantise runs in the skip schedules only");
  using Lay = DecodeLayout<D, SEQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const uint32_t sbase = smem_u32(base);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + Lay::kBar);

  const int tid = threadIdx.x;
  const Lane ln(tid);
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.group;
  const int nsplit = gridDim.x;

  int L = __ldg(p.seq_lens + b);
  const bool bad_len = (L < 0) | (L > p.max_pages * kPageSize);
  if (bad_len) L = 0;
  const int n_chunks_all = (L + kChunk - 1) / kChunk;
  int c0 = 0, c1 = n_chunks_all;
  if (!SEQ) {
    const int n128 = (L + kDecodeSplitTile - 1) / kDecodeSplitTile;
    const int per = (n128 + kDecodeSplits - 1) / kDecodeSplits;   // 128-token tiles per split
    const int sub = kDecodeSplitTile / kChunk;
    c0 = min(n_chunks_all, split * per * sub);
    c1 = min(n_chunks_all, (split + 1) * per * sub);
  }
  const int n = c1 - c0;
  const int32_t *bt = p.block_table + (size_t)b * p.max_pages;

  // validate the block-table entries this CTA will read, keeping a shared-
  // memory copy so that issuing a copy never waits on a global load
  bool bad_page = false;
  const int pg0 = c0 * (kChunk / kPageSize);
  const int pg1 = n > 0 ? (min(L, c1 * kChunk) + kPageSize - 1) / kPageSize : pg0;
  const bool bt_local = pg1 - pg0 <= Lay::kBtCap;
  int32_t *bt_s = reinterpret_cast<int32_t *>(base + Lay::kBt);
  for (int i = pg0 + tid; i < pg1; i += kThreads) {
    const int pg = __ldg(bt + i);
    bad_page |= (pg < 0) | (pg >= p.num_pages);
    if (bt_local) bt_s[i - pg0] = pg;
  }
  const int32_t *pages = bt_local ? bt_s - pg0 : bt;
  const bool any_bad = __syncthreads_or(bad_page) != 0;
  if (tid == 0 && (any_bad || bad_len))
    raise_error(p.err, any_bad ? ATTN_DEVERR_BLOCK_TABLE : ATTN_DEVERR_SEQ_LEN);

  float o_acc[D / 16][NH][4];
  float m_w[NH][2], l_w[NH][2];   // this warp's running max / this lane's partial sums, heads 8 n + cq + h
#pragma unroll
  for (int n = 0; n < NH; ++n) {
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[t][n][e] = 0.f;
    m_w[n][0] = m_w[n][1] = -INFINITY;
    l_w[n][0] = l_w[n][1] = 0.f;
  }
  bool failed = false;

  if (!any_bad && n > 0) {
    if (tid == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      for (int s = 0; s < Lay::kNumBars; ++s) mbar_init(&bars[s], 1);
      fence_barrier_init();
    }
    uint32_t qb[NH][D / 16][2];
    load_q_frags<D, NH>(qb, p.q + ((size_t)b * p.h_q + (size_t)hk * G) * D, G, ln);
    __syncthreads();
    const float sl2 = p.scale_log2;
    unsigned long long n_vis = 0, n_skip = 0;

    if (!SEQ) {
      // =============== dense: K and V of a chunk together, one pass ===============
      uint64_t *full = bars;
      int issued = 0;
      auto issue_chunk = [&](int c) {
        const int s = c % kDenseStages;
        uint8_t *ks = base + Lay::kK + 2 * s * Lay::kSlot;
        const int tok0 = (c0 + c) * kChunk;
        const int npg = (min(L - tok0, kChunk) + kPageSize - 1) / kPageSize;
        mbar_arrive_expect_tx(&full[s], 2 * npg * (D / 64) * (16 * 64 * 2));
        issue_pages<D>(&kmap, ks, &full[s], pages, tok0, L, hk, 0, 4, false);
        issue_pages<D>(&vmap, ks + Lay::kSlot, &full[s], pages, tok0, L, hk, 0, 4, false);
      };
      if (tid == 0)
        for (; issued < min(n, kDenseStages); ++issued) issue_chunk(issued);
      for (int i = 0; i < n; ++i) {
        const int s = i % kDenseStages;
        const bool ok = mbar_wait(&full[s], (i / kDenseStages) & 1, p.err);
        if (ok) {
          const uint32_t kslot = sbase + Lay::kK + 2 * s * Lay::kSlot;
          const uint32_t vslot = kslot + Lay::kSlot;
          const int tok_base = (c0 + i) * kChunk + ln.w * 16;
          float sc[NH][4], qm[NH][2];
          warp_scores<D, NH>(sc, qm, kslot, qb, tok_base, L, G, sl2, ln);
          if (tok_base < L) {
            zero_tail_rows<D>(base, vslot, tok_base, L, ln);
            warp_pv<D, NH>(o_acc, m_w, l_w, sc, qm, vslot, ln);
          }
        }
        if (__syncthreads_or(!ok)) {
          failed = true;
          break;
        }
        // every warp is done with stage s
        if (tid == 0) {
          if (issued < n) issue_chunk(issued++);
          n_vis += 1 + ((c0 + i) * kChunk + kSkipTile < L ? 1 : 0);
        }
      }
      if (failed && tid == 0)
        for (int x = issued - min(kDenseStages, issued); x < issued; ++x)
          mbar_wait(&full[x % kDenseStages], (x / kDenseStages) & 1, nullptr);
    } else {
      // =============== sequential skip schedule: score pass ahead of PV ===============
      uint64_t *kfull = bars;                         // [slot]: the chunk's K arrived
      uint64_t *vfull = bars + kSeqSlots;             // [slot]: its kept V pages arrived
      float *s_ring = reinterpret_cast<float *>(base + Lay::kS);
      float *qmax = reinterpret_cast<float *>(base + Lay::kQmax);
      float *mrun = reinterpret_cast<float *>(base + Lay::kMrun);   // [ring][tile][head]
      float p_tab = 0.f, v_tab = 0.f;
      if constexpr (QDQ) {
        p_tab = table_entry(p.p_tab, ln.lane);
        v_tab = table_entry(p.v_tab, ln.lane);
      }
      auto slot_ptr = [&](int c) { return base + Lay::kK + (c % kSeqSlots) * Lay::kSlot; };
      int k_issued = 0, v_issued = 0;                 // chunks whose K / V copies were issued
      if (tid == 0)
        for (; k_issued < min(n, kSeqSlots); ++k_issued)
          issue_pages<D>(&kmap, slot_ptr(k_issued), &kfull[k_issued % kSeqSlots], pages,
                         (c0 + k_issued) * kChunk, L, hk, 0, 4, true);
      // running max (log2 units) of head `lane` of the group, kept by lane
      // `lane` of every warp (G <= 16 <= 32), so a vote is one warp ballot
      float m_run = -INFINITY;
      uint32_t kept_bits = 0;                         // 2 bits per chunk: tiles A, B kept

      for (int i = 0; i < n + kSeqLookahead; ++i) {
        if (i < n) {
          // ---------------- score pass, chunk i ----------------
          const int sl = i % kSeqSlots;
          const bool ok = mbar_wait(&kfull[sl], (i / kSeqSlots) & 1, p.err) && !failed;
          const int tok_base = (c0 + i) * kChunk + ln.w * 16;
          float sc[NH][4], qm[NH][2];
#pragma unroll
          for (int nn = 0; nn < NH; ++nn) qm[nn][0] = qm[nn][1] = -INFINITY;
          if (ok) warp_scores<D, NH>(sc, qm, sbase + Lay::kK + sl * Lay::kSlot, qb, tok_base, L, G, sl2, ln);
          float *qx = qmax + ((i & 1) * kWarps + ln.w) * 16;
          if (ln.g == 0) {
#pragma unroll
            for (int nn = 0; nn < NH; ++nn) {
              qx[8 * nn + ln.cq] = qm[nn][0];
              qx[8 * nn + ln.cq + 1] = qm[nn][1];
            }
          }
          float *sr = s_ring + (((i % kSeqRing) * kWarps + ln.w) * 32 + ln.lane) * kRingFloats;
          if (ok) {
#pragma unroll
            for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
              for (int e = 0; e < 4; ++e) sr[nn * 4 + e] = sc[nn][e];
              sr[8 + 2 * nn] = qm[nn][0];
              sr[9 + 2 * nn] = qm[nn][1];
            }
          }
          if (__syncthreads_or(!ok)) {
            failed = true;
            break;
          }
          // every warp is done with the K of slot sl; the per-head maxima are visible
          const float *qa_x = qmax + (i & 1) * kWarps * 16;
          bool keep[2] = {true, true};
          const bool vis_b = (c0 + i) * kChunk + kSkipTile < L;
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            const bool head = ln.lane < G;
            const float tm = head ? fmaxf(qa_x[(2 * tt) * 16 + ln.lane], qa_x[(2 * tt + 1) * 16 + ln.lane])
                                  : -INFINITY;
            // a head votes skip when exp(tile max - running max) < threshold
            const bool vote = !head || (tm == -INFINITY) || (tm - m_run < p.thr_log2);
            m_run = fmaxf(m_run, tm);
            keep[tt] = !__all_sync(0xffffffffu, vote);
            if (QDQ && ln.w == 0 && head) mrun[((i % kSeqRing) * 2 + tt) * kMaxGroup + ln.lane] = m_run;
          }
          if (!vis_b) keep[1] = false;
          if (tid == 0) {
            // the V pages of the kept tiles go into the same slot (pages 0-1: tile
            // A, 2-3: tile B); the barrier phase completes even with no copy
            issue_pages<D>(&vmap, slot_ptr(i), &vfull[sl], pages, (c0 + i) * kChunk, L, hk,
                           keep[0] ? 0 : (keep[1] ? 2 : 4), keep[1] ? 4 : (keep[0] ? 2 : 4), true);
            ++v_issued;
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
        const int j = i - kSeqLookahead;
        if (j >= 0) {
          const uint32_t kb = (kept_bits >> (2 * (j & 15))) & 3u;
          const bool mine = ((kb >> (ln.w >> 1)) & 1u) != 0u;   // warps 0-1: tile A, 2-3: tile B
          const int tok_base = (c0 + j) * kChunk + ln.w * 16;
          if (mine && tok_base < L) {
            // ---------------- PV pass, chunk j ----------------
            const int sl = j % kSeqSlots;
            const bool okv = mbar_wait(&vfull[sl], (j / kSeqSlots) & 1, p.err);
            if (!okv) failed = true;
            if (okv) {
              const uint32_t vslot = sbase + Lay::kK + sl * Lay::kSlot;
              zero_tail_rows<D>(base, vslot, tok_base, L, ln);
              const float *sr = s_ring + (((j % kSeqRing) * kWarps + ln.w) * 32 + ln.lane) * kRingFloats;
              float sv[NH][4], qm[NH][2];
#pragma unroll
              for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sv[nn][e] = sr[nn * 4 + e];
                qm[nn][0] = sr[8 + 2 * nn];
                qm[nn][1] = sr[9 + 2 * nn];
              }
              if constexpr (QDQ) {
                // the walk's running max after this warp's tile (warps 0-1: tile A, 2-3: tile B)
                const float *mr = mrun + ((j % kSeqRing) * 2 + (ln.w >> 1)) * kMaxGroup;
#pragma unroll
                for (int nn = 0; nn < NH; ++nn)
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const int hh = 8 * nn + ln.cq + h;
                    qm[nn][h] = hh < G ? mr[hh] : -INFINITY;
                  }
                warp_pv_qdq<D, NH>(o_acc, m_w, l_w, sv, qm, vslot, ln, p, p_tab, v_tab);
              } else {
                warp_pv<D, NH>(o_acc, m_w, l_w, sv, qm, vslot, ln);
              }
            }
          }
          // every warp is done with slot j % kSeqSlots: it takes the K of chunk j + kSeqSlots
          if (__syncthreads_or(failed)) {
            failed = true;
            break;
          }
          if (tid == 0 && k_issued < n) {
            issue_pages<D>(&kmap, slot_ptr(k_issued), &kfull[k_issued % kSeqSlots], pages,
                           (c0 + k_issued) * kChunk, L, hk, 0, 4, true);
            ++k_issued;
          }
        }
      }
      failed = __syncthreads_or(failed) != 0;
      if (failed && tid == 0) {
        // let copies still in flight land before the shared memory goes away
        for (int c = max(0, k_issued - kSeqSlots); c < k_issued; ++c)
          mbar_wait(&kfull[c % kSeqSlots], (c / kSeqSlots) & 1, nullptr);
        for (int c = max(0, v_issued - kSeqSlots); c < v_issued; ++c)
          mbar_wait(&vfull[c % kSeqSlots], (c / kSeqSlots) & 1, nullptr);
      }
    }
    if (tid == 0 && p.skip_counts) {
      atomicAdd(p.skip_counts + 0, n_vis);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
    __syncthreads();
  }
  if constexpr (QDQ) {
    // O was accumulated in units of g over the quantised operands
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int nn = 0; nn < NH; ++nn)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[t][nn][e] *= p.qdq_out;
  }
  merge_and_store<D, NH>(base + Lay::kK, o_acc, m_w, l_w, any_bad || failed, G, b, hk, split, nsplit, SEQ, p,
                     ln);
}

// ===================== skip mode in two passes over the split schedule =====================
// For thresholds <= 1 a skipped tile never raises the running max (every row
// of it lies below the max), so the running max before a tile is the prefix
// max of all earlier tiles' maxima whether they were kept or not.  The
// decisions therefore follow from the tile maxima alone, and the sequential
// walk can be replaced by two passes over the 32-split schedule:
//   pass 1 (decode_scores_kernel): K of the split -> the group's scores
//       (fp32, log2 domain) and the per-head maxima of every 32-key tile and
//       of the whole split, written to the workspace;
//   pass 2 (decode_skip_pv_kernel): the running max entering the split is the
//       max of the earlier splits' maxima; walking its tiles in order, the
//       split takes the same decisions as the sequential walk, copies the V
//       pages and scores of kept tiles only, and leaves an (m, l, O) partial
//       for decode_combine_kernel.
// K is read once, V of kept tiles once, and the scores (4 bytes per key and
// query head) are written and read once.

// chunks in flight per CTA: two keep a pass-1 CTA at 36 KB and a pass-2 CTA at
// 46 KB of shared memory, so five or four share an SM; the per-chunk work of
// one CTA is latency-bound (barrier and dependency stalls), and more resident
// warps hid it better than deeper rings (pass 2 at 5 stages: 0.69 ms under
// ncu at 2 CTAs per SM; at 2 stages both passes 0.77 ms together)
constexpr int kScoreStages = 2;      // pass 1: K chunks
constexpr int kPvStages = 2;         // pass 2: V chunks (+ their scores)
constexpr int kTmaxCap = 1024;       // pass 2: tile maxima of a split kept in shared memory

template <int D, bool PV>
struct PassLayout {
  static constexpr int kStages = PV ? kPvStages : kScoreStages;
  static constexpr int kSlot = kChunk * D * 2;                 // K (pass 1) or V (pass 2) of a chunk
  static constexpr int kStage = kSlot + (PV ? kChunk * kMaxGroup * 4 : 0);   // + the chunk's scores
  // pass 1: [2][warp][16] 16-key maxima; pass 2: [split][G] the earlier splits' maxima
  static constexpr int kX = kStages * kStage;
  static constexpr int kTmax = kX + kDecodeSplits * kMaxGroup * 4;   // pass 2: the split's tile maxima
  // pass 2: per stage the chunk's decision bits, then per stage its chunk index
  static constexpr int kKeep = kTmax + (PV ? kTmaxCap * 4 : 0);
  // pass 2: per stage the walk's running max after each of the chunk's tiles, [stage][tile][head] (QDQ)
  static constexpr int kMrun = kKeep + 8 * kStages;
  static constexpr int kBar = kMrun + (PV ? kStages * 2 * kMaxGroup * 4 : 0);
  static constexpr int kBt = kBar + kStages * 8;
  static constexpr int kBtCap = 256;
  static constexpr int kEnd = kBt + kBtCap * 4;
  static constexpr int kMerge = kWarps * 16 * 4 * 2 + kWarps * 16 * D * 4;
  static_assert(!PV || kMerge <= kStages * kStage, "merge area fits (pass 2 merges in the ring)");
  static_assert(kStage % 1024 == 0, "stages keep the 128-byte swizzle alignment");
  static constexpr size_t kBytes = 1024 + kEnd;
};

// The split's chunk range, the sequence length (0 when out of range) and its
// block-table entries, validated and copied to shared memory when they fit.
struct SplitRange {
  int L, c0, c1;
  const int32_t *pages;   // indexed by the sequence's page number
  bool dead;              // a block-table entry of the range is out of bounds
};

// `extra(L, c0, c1)` runs before the block-table loads and before the barrier
// that publishes them, so loads it issues share their round trip.
template <typename Extra>
ATTN_DEVICE SplitRange split_range(const DecodeParams &p, int b, int split, int32_t *bt_s, int bt_cap,
                                   Extra extra, int L) {
  SplitRange r;
  const bool bad_len = (L < 0) | (L > p.max_pages * kPageSize);
  if (bad_len) L = 0;
  const int n_chunks_all = (L + kChunk - 1) / kChunk;
  const int n128 = (L + kDecodeSplitTile - 1) / kDecodeSplitTile;
  const int per = (n128 + kDecodeSplits - 1) / kDecodeSplits;
  const int sub = kDecodeSplitTile / kChunk;
  r.L = L;
  r.c0 = min(n_chunks_all, split * per * sub);
  r.c1 = min(n_chunks_all, (split + 1) * per * sub);
  extra(L, r.c0, r.c1);
  const int32_t *bt = p.block_table + (size_t)b * p.max_pages;
  const int pg0 = r.c0 * (kChunk / kPageSize);
  const int pg1 = r.c1 > r.c0 ? (min(L, r.c1 * kChunk) + kPageSize - 1) / kPageSize : pg0;
  const bool local = pg1 - pg0 <= bt_cap;
  bool bad_page = false;
  for (int i = pg0 + (int)threadIdx.x; i < pg1; i += kThreads) {
    const int pg = __ldg(bt + i);
    bad_page |= (pg < 0) | (pg >= p.num_pages);
    if (local) bt_s[i - pg0] = pg;
  }
  r.pages = local ? bt_s - pg0 : bt;
  r.dead = __syncthreads_or(bad_page) != 0;
  if (threadIdx.x == 0 && (r.dead || bad_len))
    raise_error(p.err, r.dead ? ATTN_DEVERR_BLOCK_TABLE : ATTN_DEVERR_SEQ_LEN);
  return r;
}

template <int D, int NH>
__global__ void __launch_bounds__(kThreads) decode_scores_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                 DecodeParams p) {
  using Lay = PassLayout<D, false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const uint32_t sbase = smem_u32(base);
  uint64_t *full = reinterpret_cast<uint64_t *>(base + Lay::kBar);
  float *qx = reinterpret_cast<float *>(base + Lay::kX);
  const int tid = threadIdx.x;
  const Lane ln(tid);
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.group;
  const SplitRange r = split_range(p, b, split, reinterpret_cast<int32_t *>(base + Lay::kBt), Lay::kBtCap,
                                   [](int, int, int) {}, __ldg(p.seq_lens + b));
  const int n = r.c1 - r.c0;
  const size_t seq = (size_t)b * p.h_kv + hk;
  float *S = p.ws_s + seq * (size_t)p.s_stride * G;          // [token][G]
  float *tmax = p.ws_tmax + seq * (size_t)p.kt_max * G;     // [tile][G]
  float smax = -INFINITY;   // thread (tt, h) = tid (tt * G + h): head h's max over tiles tt of each chunk
  if (!r.dead && n > 0) {
    if (tid == 0) {
      tma_prefetch_desc(&kmap);
      for (int s = 0; s < Lay::kStages; ++s) mbar_init(&full[s], 1);
      fence_barrier_init();
    }
    uint32_t qb[NH][D / 16][2];
    load_q_frags<D, NH>(qb, p.q + ((size_t)b * p.h_q + (size_t)hk * G) * D, G, ln);
    __syncthreads();
    int issued = 0;
    auto issue = [&](int c) {
      const int s = c % Lay::kStages;
      issue_pages<D>(&kmap, base + s * Lay::kStage, &full[s], r.pages, (r.c0 + c) * kChunk, r.L, hk, 0, 4,
                     true);
    };
    if (tid == 0)
      for (; issued < min(n, Lay::kStages); ++issued) issue(issued);
    bool failed = false;
    for (int i = 0; i < n; ++i) {
      const int s = i % Lay::kStages;
      const bool ok = mbar_wait(&full[s], (i / Lay::kStages) & 1, p.err);
      if (ok) {
        const int tok_base = (r.c0 + i) * kChunk + ln.w * 16;
        float sc[NH][4], qm[NH][2];
        warp_scores<D, NH>(sc, qm, sbase + s * Lay::kStage, qb, tok_base, r.L, G, p.scale_log2, ln);
#pragma unroll
        for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = tok_base + ln.g + 8 * (e >> 1);
            const int h = 8 * nn + ln.cq + (e & 1);
            if (t < r.L && h < G) S[(size_t)t * G + h] = sc[nn][e];
          }
          if (ln.g == 0) {
            qx[((i & 1) * kWarps + ln.w) * 16 + 8 * nn + ln.cq] = qm[nn][0];
            qx[((i & 1) * kWarps + ln.w) * 16 + 8 * nn + ln.cq + 1] = qm[nn][1];
          }
        }
      }
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // every warp is done with stage s; chunk i's 16-key maxima are visible
      if (tid == 0 && issued < n) issue(issued++);
      if (tid < 2 * G) {
        const int tt = tid / G, h = tid % G;
        const float *x = qx + (i & 1) * kWarps * 16;
        const float tm = fmaxf(x[(2 * tt) * 16 + h], x[(2 * tt + 1) * 16 + h]);
        const int tile = 2 * (r.c0 + i) + tt;
        if (tile * kSkipTile < r.L) tmax[(size_t)tile * G + h] = tm;
        smax = fmaxf(smax, tm);
      }
    }
    if (failed && tid == 0)
      for (int x = issued - min(Lay::kStages, issued); x < issued; ++x)
        mbar_wait(&full[x % Lay::kStages], (x / Lay::kStages) & 1, nullptr);
  }
  if (tid < 32) {
    // lanes h and G + h hold head h's maxima over the chunks' first and second tiles
    const float other = __shfl_sync(0xffffffffu, smax, (tid + G) & 31);
    if (tid < G) p.ws_smax[(seq * kDecodeSplits + split) * G + tid] = fmaxf(smax, other);
  }
}

// ORs bits [u0, u1) of a bit mask in global memory, a word at a time.
ATTN_DEVICE void or_bit_range(uint32_t *mask, long long u0, long long u1) {
  while (u0 < u1) {
    const long long w = u0 >> 5;
    const int lo = (int)(u0 & 31);
    const long long span = u1 - (w << 5);
    const int hi = span < 32 ? (int)span : 32;
    const uint32_t bits = (hi == 32 ? 0xffffffffu : ((1u << hi) - 1u)) & ~((1u << lo) - 1u);
    atomicOr(mask + w, bits);
    u0 = (w + 1) << 5;
  }
}

template <int D, int NH, bool QDQ>
__global__ void __launch_bounds__(kThreads) decode_skip_pv_kernel(const __grid_constant__ CUtensorMap vmap,
                                                                  DecodeParams p) {
  using Lay = PassLayout<D, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const uint32_t sbase = smem_u32(base);
  uint64_t *full = reinterpret_cast<uint64_t *>(base + Lay::kBar);
  float *tm_s = reinterpret_cast<float *>(base + Lay::kTmax);
  uint32_t *keep_s = reinterpret_cast<uint32_t *>(base + Lay::kKeep);
  float *mrun_s = reinterpret_cast<float *>(base + Lay::kMrun);   // [stage][tile][head]
  const int tid = threadIdx.x;
  const Lane ln(tid);
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.group;
  const size_t seq = (size_t)b * p.h_kv + hk;
  const float *S = p.ws_s + seq * (size_t)p.s_stride * G;
  const float *tmax = p.ws_tmax + seq * (size_t)p.kt_max * G;

  // with the block-table entries, in the same round trip: the split's tile
  // maxima and the earlier splits' maxima, to shared memory
  float *sm_s = reinterpret_cast<float *>(base + Lay::kX);   // [split][G], this and earlier splits
  const SplitRange r = split_range(
      p, b, split, reinterpret_cast<int32_t *>(base + Lay::kBt), Lay::kBtCap, [&](int L, int c0, int c1) {
        const int nt = max(0, min((L + kSkipTile - 1) / kSkipTile, 2 * c1) - 2 * c0);
        const int ntm = (2 * (c1 - c0) * G <= kTmaxCap) ? nt * G : 0;
        const int nsm = (split + 1) * G;   // (with this split's own)
        const float *tsrc = tmax + (size_t)2 * c0 * G;
        const float *ssrc = p.ws_smax + seq * kDecodeSplits * G;
        const float a = tid < ntm ? tsrc[tid] : 0.f;
        const float c = tid < nsm ? ssrc[tid] : 0.f;
        if (tid < ntm) tm_s[tid] = a;
        if (tid < nsm) sm_s[tid] = c;
        for (int x = tid + kThreads; x < ntm; x += kThreads) tm_s[x] = tsrc[x];
        for (int x = tid + kThreads; x < nsm; x += kThreads) sm_s[x] = ssrc[x];
      },
      __ldg(p.seq_lens + b));
  const int n = r.c1 - r.c0;
  const bool tm_local = 2 * n * G <= kTmaxCap;

  float o_acc[D / 16][NH][4];
  float m_w[NH][2], l_w[NH][2];
#pragma unroll
  for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[t][nn][e] = 0.f;
    m_w[nn][0] = m_w[nn][1] = -INFINITY;
    l_w[nn][0] = l_w[nn][1] = 0.f;
  }
  bool failed = false;
  if (!r.dead && n > 0) {
    if (tid == 0) {
      tma_prefetch_desc(&vmap);
      for (int s = 0; s < Lay::kStages; ++s) mbar_init(&full[s], 1);
      fence_barrier_init();
    }
    // warp 0 takes the decisions (lane h: head h) and issues the copies
    const bool head = ln.lane < G;
    float p_tab = 0.f, v_tab = 0.f;
    if constexpr (QDQ) {
      p_tab = table_entry(p.p_tab, ln.lane);
      v_tab = table_entry(p.v_tab, ln.lane);
    }
    float m_run = -INFINITY;   // head lane's running max entering the next tile
    unsigned long long n_vis = 0, n_skip = 0;
    // A split whose maximum (per head, from the first pass) is below the
    // threshold relative to the earlier splits' maximum has every tile
    // skipped: the running max entering any of its tiles is at least that,
    // and no tile max exceeds the split's.  It is settled here, with no ring:
    // its tiles are counted and marked skipped, and it leaves an empty partial.
    bool all_skipped = true;
    if (ln.w == 0) {
      for (int h = 0; h < G; ++h) {
        const float mp = warp_max(ln.lane < split ? sm_s[ln.lane * G + h] : -INFINITY);
        if (ln.lane == h) m_run = mp;   // the earlier splits' maximum
        const float mine = sm_s[split * G + h];
        all_skipped = all_skipped && (mine == -INFINITY || mine - mp < p.thr_log2);
      }
    }
    if (__syncthreads_and(all_skipped)) {   // (also publishes the barrier init)
      const int t0 = 2 * r.c0, t1 = min((r.L + kSkipTile - 1) / kSkipTile, 2 * r.c1);
      if (tid == 0 && t1 > t0) {
        if (p.skip_counts) {
          atomicAdd(p.skip_counts + 0, (unsigned long long)(t1 - t0));
          atomicAdd(p.skip_counts + 1, (unsigned long long)(t1 - t0));
        }
        if (p.skip_mask)
          or_bit_range(p.skip_mask, (long long)seq * p.kt_max + t0, (long long)seq * p.kt_max + t1);
      }
      if (tid < G) {
        const size_t row = ((size_t)b * p.h_q + (size_t)hk * G + tid) * kDecodeSplits + split;
        p.ws_ml[row * 2 + 0] = -INFINITY;
        p.ws_ml[row * 2 + 1] = 0.f;
      }
      return;
    }
    // decide() leaves the head lane's running max after each of the chunk's
    // tiles in dm[] (the reference max of the quantised P)
    float dm[2] = {-INFINITY, -INFINITY};
    auto decide = [&](int c) -> uint32_t {
      uint32_t kb = 0;
#pragma unroll
      for (int tt = 0; tt < 2; ++tt) {
        const int tile = 2 * (r.c0 + c) + tt;
        const bool vis = tile * kSkipTile < r.L;
        const float tm = (vis && head) ? (tm_local ? tm_s[(2 * c + tt) * G + ln.lane]
                                                   : tmax[(size_t)tile * G + ln.lane])
                                       : -INFINITY;
        // a head votes skip when exp(tile max - running max) < threshold
        const bool vote = !head || tm == -INFINITY || (tm - m_run < p.thr_log2);
        m_run = fmaxf(m_run, tm);
        dm[tt] = m_run;
        const bool kept = vis && !__all_sync(0xffffffffu, vote);
        if (kept) kb |= 1u << tt;
        if (vis) {
          ++n_vis;
          if (!kept) {
            ++n_skip;
            if (p.skip_mask && ln.lane == 0) {
              const long long unit = (long long)seq * p.kt_max + tile;
              atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
            }
          }
        }
      }
      return kb;
    };
    auto issue = [&](int i, int c, uint32_t kb) {   // lane 0 of warp 0: ring position i, chunk c
      const int s = i % Lay::kStages;
      uint8_t *stage = base + s * Lay::kStage;
      const int tok0 = (r.c0 + c) * kChunk;
      const int npg = (min(r.L - tok0, kChunk) + kPageSize - 1) / kPageSize;
      // pages 0-1 hold tile A, 2-3 tile B
      const int lo = (kb & 1u) ? 0 : ((kb & 2u) ? 2 : 4);
      const int hi = min(npg, (kb & 2u) ? 4 : ((kb & 1u) ? 2 : 0));
      const uint32_t sbytes = kb ? kChunk * G * 4 : 0u;
      keep_s[s] = kb;
      keep_s[Lay::kStages + s] = (uint32_t)c;
      mbar_arrive_expect_tx(&full[s], max(0, hi - lo) * (D / 64) * (16 * 64 * 2) + sbytes);
      issue_pages<D>(&vmap, stage, &full[s], r.pages, tok0, r.L, hk, lo, hi, false);
      if (sbytes) bulk_load(stage + Lay::kSlot, S + (size_t)tok0 * G, sbytes, &full[s]);
    };
    // Warp 0 decides the chunks in tile order and puts only the kept ones in
    // the ring, each marked when no kept chunk follows (it decides one kept
    // chunk ahead): a skipped chunk costs its decision, taken while the other
    // warps work on earlier chunks, not a round of the ring.  A split with
    // no kept chunk gets one end entry.
    constexpr uint32_t kLast = 4u, kEndEntry = 0xffffffffu;
    int next_c = 0;              // warp 0: the next chunk to decide
    int pend_c = 0;              // warp 0: the next kept chunk and its tile bits (0: none)
    uint32_t pend_kb = 0;
    float pend_m[2] = {-INFINITY, -INFINITY};   // and its running maxima (QDQ)
    bool more = true;            // warp 0: the last entry is not issued yet
    auto find_kept = [&]() {
      pend_kb = 0;
      while (pend_kb == 0 && next_c < n) {
        pend_c = next_c++;
        pend_kb = decide(pend_c);
      }
      pend_m[0] = dm[0];
      pend_m[1] = dm[1];
    };
    auto next_issue = [&](int i) {   // warp 0: ring position i
      const int c = pend_c;
      const uint32_t kb = pend_kb;
      if constexpr (QDQ) {
        if (kb && head) {
          mrun_s[((i % Lay::kStages) * 2 + 0) * kMaxGroup + ln.lane] = pend_m[0];
          mrun_s[((i % Lay::kStages) * 2 + 1) * kMaxGroup + ln.lane] = pend_m[1];
        }
        __syncwarp();
      }
      if (kb) find_kept();
      if (ln.lane == 0) {
        if (kb) {
          issue(i, c, kb | (pend_kb ? 0u : kLast));
        } else {
          keep_s[i % Lay::kStages] = kEndEntry;
          mbar_arrive(&full[i % Lay::kStages]);
        }
      }
      more = kb != 0 && pend_kb != 0;
    };
    int issued = 0;
    if (ln.w == 0) {
      find_kept();
      for (; more && issued < Lay::kStages; ++issued) next_issue(issued);
    }
    for (int i = 0;; ++i) {
      const int s = i % Lay::kStages;
      const bool ok = mbar_wait(&full[s], (i / Lay::kStages) & 1, p.err);
      bool ended = false;
      if (ok) {
        const uint32_t kb = keep_s[s];
        ended = kb == kEndEntry || (kb & kLast);
        const int tok_base = (r.c0 + (int)keep_s[Lay::kStages + s]) * kChunk + ln.w * 16;
        if (kb != kEndEntry && ((kb >> (ln.w >> 1)) & 1u) && tok_base < r.L) {
          const uint32_t vslot = sbase + s * Lay::kStage;
          const float *ss = reinterpret_cast<const float *>(base + s * Lay::kStage + Lay::kSlot);
          float sc[NH][4], qm[NH][2];
#pragma unroll
          for (int nn = 0; nn < NH; ++nn) {
            qm[nn][0] = qm[nn][1] = -INFINITY;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int tl = ln.w * 16 + ln.g + 8 * (e >> 1);
              const int h = 8 * nn + ln.cq + (e & 1);
              const float v = (tok_base - ln.w * 16 + tl < r.L && h < G) ? ss[tl * G + h] : -INFINITY;
              sc[nn][e] = v;
              qm[nn][e & 1] = fmaxf(qm[nn][e & 1], v);
            }
            if constexpr (!QDQ) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int o = 4; o < 32; o <<= 1)
                  qm[nn][h] = fmaxf(qm[nn][h], __shfl_xor_sync(0xffffffffu, qm[nn][h], o));
            }
          }
          zero_tail_rows<D>(base, vslot, tok_base, r.L, ln);
          if constexpr (QDQ) {
            // the walk's running max after this warp's tile (warps 0-1: tile A, 2-3: tile B)
            const float *mr = mrun_s + (s * 2 + (ln.w >> 1)) * kMaxGroup;
#pragma unroll
            for (int nn = 0; nn < NH; ++nn)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int hh = 8 * nn + ln.cq + h;
                qm[nn][h] = hh < G ? mr[hh] : -INFINITY;
              }
            warp_pv_qdq<D, NH>(o_acc, m_w, l_w, sc, qm, vslot, ln, p, p_tab, v_tab);
          } else {
            warp_pv<D, NH>(o_acc, m_w, l_w, sc, qm, vslot, ln);
          }
        }
      }
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      if (ended) break;
      // every warp is done with stage s
      if (ln.w == 0 && more) {
        next_issue(issued);
        ++issued;
      }
    }
    if (failed && tid == 0)
      for (int x = issued - min(Lay::kStages, issued); x < issued; ++x)
        mbar_wait(&full[x % Lay::kStages], (x / Lay::kStages) & 1, nullptr);
    if (tid == 0 && p.skip_counts) {
      atomicAdd(p.skip_counts + 0, n_vis);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
    __syncthreads();
  }
  if constexpr (QDQ) {
    // O was accumulated in units of g over the quantised operands
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int nn = 0; nn < NH; ++nn)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[t][nn][e] *= p.qdq_out;
  }
  merge_and_store<D, NH>(base, o_acc, m_w, l_w, r.dead || failed, G, b, hk, split, kDecodeSplits, false, p,
                         ln);
}

// ---------------------------------------------------------------------------
// Skip mode in one pass over the split schedule
// ---------------------------------------------------------------------------
// One CTA per (split, kv-head, sequence) computes its split's scores into
// shared memory (K chunks through the ring), publishes the split's maximum
// per head, takes the earlier splits' maxima from the CTAs that computed them,
// and then walks its 32-key tiles with the running max they give, copying the
// V chunks of kept tiles through the same ring.  The decisions are the two
// passes' (and the sequential walk's); the scores never leave the SM.  CTAs
// take their split from a ticket counter in start order, splits innermost,
// so every split a CTA waits for belongs to a CTA that started before it.
// (Parking the scores in tensor memory instead, with a third ring stage in
// the shared memory that frees, measured slower.)
constexpr int kOneStages = 2;
constexpr int kOneBtCap = 256;

struct OnePassLayout {
  size_t ring, sc, tm, qx, bt, keep, bar, total;
  __host__ __device__ OnePassLayout(int d, int group, int split_keys) {
    const size_t slot = (size_t)kChunk * d * 2;
    ring = 0;
    sc = ring + kOneStages * slot;                                   // [split_keys][G] scores
    tm = sc + (((size_t)split_keys * group * 4 + 15) & ~size_t(15)); // [split_keys / 32][G] tile maxima
    qx = tm + (((size_t)(split_keys / kSkipTile) * group * 4 + 15) & ~size_t(15));   // [chunk][warp][16]
    bt = qx + (size_t)(split_keys / kChunk) * kWarps * 16 * 4;       // block-table entries
    keep = bt + kOneBtCap * 4;                                       // [stage] bits, [stage] chunk
    bar = keep + 2 * kOneStages * 4;                                 // [stage] mbarriers
    total = bar + kOneStages * 8;
  }
};

template <int D, int NH>
__global__ void __launch_bounds__(kThreads) decode_one_pass_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                   const __grid_constant__ CUtensorMap vmap,
                                                                   DecodeParams p) {
  constexpr int kSlot = kChunk * D * 2;
  constexpr int S = kOneStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = align1024(smem_raw);
  const uint32_t sbase = smem_u32(base);
  const int G = p.group;
  const OnePassLayout lay(D, G, p.split_keys);
  float *sc_s = reinterpret_cast<float *>(base + lay.sc);
  float *tm_s = reinterpret_cast<float *>(base + lay.tm);
  float *qx = reinterpret_cast<float *>(base + lay.qx);
  uint32_t *keep_s = reinterpret_cast<uint32_t *>(base + lay.keep);
  uint64_t *full = reinterpret_cast<uint64_t *>(base + lay.bar);
  const int tid = threadIdx.x;
  const Lane ln(tid);
  __shared__ int ticket;
  if (tid == 0) ticket = (int)atomicAdd(p.ws_ticket, 1u);
  __syncthreads();
  const int split = ticket % kDecodeSplits;
  const int hk = (ticket / kDecodeSplits) % p.h_kv;
  const int b = ticket / (kDecodeSplits * p.h_kv);
  const size_t seq = (size_t)b * p.h_kv + hk;
  unsigned long long *pub = p.ws_pub + seq * kDecodeSplits * G;   // [split][G]

  const SplitRange r = split_range(p, b, split, reinterpret_cast<int32_t *>(base + lay.bt), kOneBtCap,
                                   [](int, int, int) {}, __ldg(p.seq_lens + b));
  const int n = r.c1 - r.c0;
  bool failed = false;
  float smax = -INFINITY;   // thread (tt, h) = tid (tt * G + h): head h's max over tiles tt of each chunk

  // ---- first half: the split's scores and tile maxima (K chunks) ----
  if (!r.dead && n > 0) {
    if (tid == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      for (int st = 0; st < S; ++st) mbar_init(&full[st], 1);
      fence_barrier_init();
    }
    uint32_t qb[NH][D / 16][2];
    load_q_frags<D, NH>(qb, p.q + ((size_t)b * p.h_q + (size_t)hk * G) * D, G, ln);
    __syncthreads();
    int issued = 0;
    auto issue_k = [&](int c) {
      const int st = c % S;
      issue_pages<D>(&kmap, base + st * kSlot, &full[st], r.pages, (r.c0 + c) * kChunk, r.L, hk, 0, 4, true);
    };
    if (tid == 0)
      for (; issued < min(n, S); ++issued) issue_k(issued);
    for (int i = 0; i < n; ++i) {
      const int st = i % S;
      const bool ok = mbar_wait(&full[st], (i / S) & 1, p.err);
      if (ok) {
        const int tok_base = (r.c0 + i) * kChunk + ln.w * 16;
        float sc[NH][4], qm[NH][2];
        warp_scores<D, NH>(sc, qm, sbase + st * kSlot, qb, tok_base, r.L, G, p.scale_log2, ln);
#pragma unroll
        for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tl = ln.w * 16 + ln.g + 8 * (e >> 1);
            const int h = 8 * nn + ln.cq + (e & 1);
            if (h < G) sc_s[((size_t)i * kChunk + tl) * G + h] = sc[nn][e];
          }
          if (ln.g == 0) {
            qx[(i * kWarps + ln.w) * 16 + 8 * nn + ln.cq] = qm[nn][0];
            qx[(i * kWarps + ln.w) * 16 + 8 * nn + ln.cq + 1] = qm[nn][1];
          }
        }
      }
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      // every warp is done with stage st
      if (tid == 0 && issued < n) issue_k(issued++);
    }
    // the 32-key tile maxima from the warps' 16-key ones, once every chunk is
    // in (off the per-chunk path); written and read by warp 0 only
    if (!failed && tid < 2 * G) {
      const int tt = tid / G, h = tid % G;
      for (int i = 0; i < n; ++i) {
        const float *x = qx + i * kWarps * 16;
        const float tmv = fmaxf(x[(2 * tt) * 16 + h], x[(2 * tt + 1) * 16 + h]);
        tm_s[(2 * i + tt) * G + h] = tmv;
        smax = fmaxf(smax, tmv);
      }
    }
    __syncwarp();
    if (failed && tid == 0)
      for (int x = issued - min(S, issued); x < issued; ++x) mbar_wait(&full[x % S], (x / S) & 1, nullptr);
  }

  // ---- publish this split's maximum per head (every split, so that none waits in vain) ----
  float own = -INFINITY;   // warp 0, lane h < G: head h's maximum over this split
  if (tid < 32) {
    const float other = __shfl_sync(0xffffffffu, smax, (tid + G) & 31);
    own = fmaxf(smax, other);
    if (tid < G) {
      const unsigned long long w = (1ull << 32) | __float_as_uint(own);
      asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(pub + split * G + tid), "l"(w) : "memory");
    }
  }

  float o_acc[D / 16][NH][4];
  float m_w[NH][2], l_w[NH][2];
#pragma unroll
  for (int nn = 0; nn < NH; ++nn) {
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o_acc[t][nn][e] = 0.f;
    m_w[nn][0] = m_w[nn][1] = -INFINITY;
    l_w[nn][0] = l_w[nn][1] = 0.f;
  }

  if (!r.dead && n > 0 && !failed) {
    // ---- the earlier splits' maxima (lane x waits for split x) ----
    float m_run = -INFINITY;   // warp 0, head lane: the running max entering the next tile
    bool all_skipped = true;
    if (ln.w == 0) {
      float v[kMaxGroup];
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) v[h] = -INFINITY;
      bool got = true;
      if (ln.lane < split) {
        const uint64_t t0 = globaltimer_ns();
        for (int h = 0; h < G; ++h) {
          unsigned long long w = 0;
          for (uint32_t it = 0;; ++it) {
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(pub + ln.lane * G + h) : "memory");
            if ((w >> 32) != 0ull) break;
            if (it >= kSpinLimit || globaltimer_ns() - t0 > 1000000000ull) {
              got = false;
              break;
            }
            __nanosleep(64);
          }
          if (!got) break;
          const float x = __uint_as_float((uint32_t)w);
#pragma unroll
          for (int hh = 0; hh < kMaxGroup; ++hh)
            if (hh == h) v[hh] = x;
        }
      }
      if (!__all_sync(0xffffffffu, got)) {
        if (ln.lane == 0) raise_error(p.err, ATTN_DEVERR_TIMEOUT);
        failed = true;
      }
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= G) break;
        const float mp = warp_max(v[h]);
        if (ln.lane == h) m_run = mp;
      }
      // every tile of the split is skipped when its maximum is below the
      // threshold against the earlier splits' for every head
      all_skipped = __all_sync(0xffffffffu, ln.lane >= G || own == -INFINITY || own - m_run < p.thr_log2);
    }
    failed = __syncthreads_or(failed);
    if (!failed && __syncthreads_and(all_skipped)) {
      const int t0 = 2 * r.c0, t1 = min((r.L + kSkipTile - 1) / kSkipTile, 2 * r.c1);
      if (tid == 0 && t1 > t0) {
        if (p.skip_counts) {
          atomicAdd(p.skip_counts + 0, (unsigned long long)(t1 - t0));
          atomicAdd(p.skip_counts + 1, (unsigned long long)(t1 - t0));
        }
        if (p.skip_mask)
          or_bit_range(p.skip_mask, (long long)seq * p.kt_max + t0, (long long)seq * p.kt_max + t1);
      }
      if (tid < G) {
        const size_t row = ((size_t)b * p.h_q + (size_t)hk * G + tid) * kDecodeSplits + split;
        p.ws_ml[row * 2 + 0] = -INFINITY;
        p.ws_ml[row * 2 + 1] = 0.f;
      }
      return;
    }

    // ---- second half: the kept tiles' P.V (V chunks through the same ring) ----
    if (!failed) {
      const bool head = ln.lane < G;
      unsigned long long n_vis = 0, n_skip = 0;
      auto decide = [&](int c) -> uint32_t {
        uint32_t kb = 0;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const int tile = 2 * (r.c0 + c) + tt;
          const bool vis = tile * kSkipTile < r.L;
          const float tmv = (vis && head) ? tm_s[(2 * c + tt) * G + ln.lane] : -INFINITY;
          // a head votes skip when exp(tile max - running max) < threshold
          const bool vote = !head || tmv == -INFINITY || (tmv - m_run < p.thr_log2);
          m_run = fmaxf(m_run, tmv);
          const bool kept = vis && !__all_sync(0xffffffffu, vote);
          if (kept) kb |= 1u << tt;
          if (vis) {
            ++n_vis;
            if (!kept) {
              ++n_skip;
              if (p.skip_mask && ln.lane == 0) {
                const long long unit = (long long)seq * p.kt_max + tile;
                atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
              }
            }
          }
        }
        return kb;
      };
      // ring positions continue after the n K chunks
      auto issue_v = [&](int i, int c, uint32_t kb) {   // lane 0 of warp 0
        const int pos = n + i, st = pos % S;
        const int tok0 = (r.c0 + c) * kChunk;
        const int npg = (min(r.L - tok0, kChunk) + kPageSize - 1) / kPageSize;
        // pages 0-1 hold tile A, 2-3 tile B
        const int lo = (kb & 1u) ? 0 : ((kb & 2u) ? 2 : 4);
        const int hi = min(npg, (kb & 2u) ? 4 : ((kb & 1u) ? 2 : 0));
        keep_s[st] = kb;
        keep_s[S + st] = (uint32_t)c;
        mbar_arrive_expect_tx(&full[st], max(0, hi - lo) * (D / 64) * (16 * 64 * 2));
        issue_pages<D>(&vmap, base + st * kSlot, &full[st], r.pages, tok0, r.L, hk, lo, hi, false);
      };
      // warp 0 decides the chunks in tile order and rings only the kept ones,
      // the last marked (it decides one kept chunk ahead); a split with none
      // kept gets one end entry
      constexpr uint32_t kLast = 4u, kEndEntry = 0xffffffffu;
      int next_c = 0, pend_c = 0;
      uint32_t pend_kb = 0;
      bool more = true;
      auto find_kept = [&]() {
        pend_kb = 0;
        while (pend_kb == 0 && next_c < n) {
          pend_c = next_c++;
          pend_kb = decide(pend_c);
        }
      };
      auto next_issue = [&](int i) {
        const int c = pend_c;
        const uint32_t kb = pend_kb;
        if (kb) find_kept();
        if (ln.lane == 0) {
          if (kb) {
            issue_v(i, c, kb | (pend_kb ? 0u : kLast));
          } else {
            keep_s[(n + i) % S] = kEndEntry;
            mbar_arrive(&full[(n + i) % S]);
          }
        }
        more = kb != 0 && pend_kb != 0;
      };
      int issued = 0;
      if (ln.w == 0) {
        find_kept();
        for (; more && issued < S; ++issued) next_issue(issued);
      }
      for (int i = 0;; ++i) {
        const int pos = n + i, st = pos % S;
        const bool ok = mbar_wait(&full[st], (pos / S) & 1, p.err);
        bool ended = false;
        if (ok) {
          const uint32_t kb = keep_s[st];
          ended = kb == kEndEntry || (kb & kLast);
          const int c = (int)keep_s[S + st];
          const int tok_base = (r.c0 + c) * kChunk + ln.w * 16;
          if (kb != kEndEntry && ((kb >> (ln.w >> 1)) & 1u) && tok_base < r.L) {
            const uint32_t vslot = sbase + st * kSlot;
            const float *ss = sc_s + (size_t)c * kChunk * G;
            float sc[NH][4], qm[NH][2];
#pragma unroll
            for (int nn = 0; nn < NH; ++nn) {
              qm[nn][0] = qm[nn][1] = -INFINITY;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int tl = ln.w * 16 + ln.g + 8 * (e >> 1);
                const int h = 8 * nn + ln.cq + (e & 1);
                const float v = (tok_base - ln.w * 16 + tl < r.L && h < G) ? ss[tl * G + h] : -INFINITY;
                sc[nn][e] = v;
                qm[nn][e & 1] = fmaxf(qm[nn][e & 1], v);
              }
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int o = 4; o < 32; o <<= 1)
                  qm[nn][h] = fmaxf(qm[nn][h], __shfl_xor_sync(0xffffffffu, qm[nn][h], o));
            }
            zero_tail_rows<D>(base, vslot, tok_base, r.L, ln);
            warp_pv<D, NH>(o_acc, m_w, l_w, sc, qm, vslot, ln);
          }
        }
        if (__syncthreads_or(!ok)) {
          failed = true;
          break;
        }
        if (ended) break;
        // every warp is done with stage st
        if (ln.w == 0 && more) {
          next_issue(issued);
          ++issued;
        }
      }
      if (failed && tid == 0)
        for (int x = issued - min(S, issued); x < issued; ++x)
          mbar_wait(&full[(n + x) % S], ((n + x) / S) & 1, nullptr);
      if (tid == 0 && p.skip_counts) {
        atomicAdd(p.skip_counts + 0, n_vis);
        atomicAdd(p.skip_counts + 1, n_skip);
      }
      __syncthreads();
    }
  }
  merge_and_store<D, NH>(base, o_acc, m_w, l_w, r.dead || failed, G, b, hk, split, kDecodeSplits, false, p,
                         ln);
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

template <int D, bool SEQ, int NH, bool QDQ>
cudaError_t launch_k(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
  const size_t smem = DecodeLayout<D, SEQ>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, SEQ, NH, QDQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(SEQ ? 1 : kDecodeSplits, p.h_kv, p.batch);
  decode_kernel<D, SEQ, NH, QDQ><<<grid, kThreads, smem, stream>>>(kmap, vmap, p);
  return cudaGetLastError();
}

// one n-tile of 8 heads for groups of up to 8 query heads, two up to 16
template <int D, bool SEQ, bool QDQ>
cudaError_t launch_g(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
  return p.group <= 8 ? launch_k<D, SEQ, 1, QDQ>(p, kmap, vmap, stream)
                      : launch_k<D, SEQ, 2, QDQ>(p, kmap, vmap, stream);
}

template <int D, int NH, bool QDQ>
cudaError_t launch_two_pass(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                            cudaStream_t stream) {
  const size_t s1 = PassLayout<D, false>::kBytes, s2 = PassLayout<D, true>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(decode_scores_kernel<D, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)s1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(decode_skip_pv_kernel<D, NH, QDQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)s2);
  if (e != cudaSuccess) return e;
  dim3 grid(kDecodeSplits, p.h_kv, p.batch);
  decode_scores_kernel<D, NH><<<grid, kThreads, s1, stream>>>(kmap, p);
  decode_skip_pv_kernel<D, NH, QDQ><<<grid, kThreads, s2, stream>>>(vmap, p);
  return cudaGetLastError();
}

template <int D, bool QDQ>
cudaError_t launch_two_pass_g(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                              cudaStream_t stream) {
  return p.group <= 8 ? launch_two_pass<D, 1, QDQ>(p, kmap, vmap, stream)
                      : launch_two_pass<D, 2, QDQ>(p, kmap, vmap, stream);
}

template <int D, int NH>
cudaError_t launch_one_pass(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                            cudaStream_t stream) {
  const size_t smem = 1024 + OnePassLayout(D, p.group, p.split_keys).total;
  cudaError_t e = cudaFuncSetAttribute(decode_one_pass_kernel<D, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((long long)p.batch * p.h_kv * kDecodeSplits);
  decode_one_pass_kernel<D, NH><<<grid, kThreads, smem, stream>>>(kmap, vmap, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
  const bool qdq = p.p_qdq || p.v_qdq;
  if (p.sequential == 3) {
    const cudaError_t e1 = p.group <= 8 ? launch_one_pass<D, 1>(p, kmap, vmap, stream)
                                        : launch_one_pass<D, 2>(p, kmap, vmap, stream);
    if (e1 != cudaSuccess) return e1;
    const long long rows = (long long)p.batch * p.h_q;
    decode_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p);
    return cudaGetLastError();
  }
  if (p.sequential == 1)
    return qdq ? launch_g<D, true, true>(p, kmap, vmap, stream) : launch_g<D, true, false>(p, kmap, vmap, stream);
  cudaError_t e = p.sequential == 2
                      ? (qdq ? launch_two_pass_g<D, true>(p, kmap, vmap, stream)
                             : launch_two_pass_g<D, false>(p, kmap, vmap, stream))
                      : launch_g<D, false, false>(p, kmap, vmap, stream);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)p.batch * p.h_q;
  decode_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t decode_one_pass_smem(int d, int group, int split_keys) {
  const size_t bytes = 1024 + OnePassLayout(d, group, split_keys).total;
  // the second half's merge reuses the ring and the scores
  const size_t merge = (size_t)kWarps * 16 * 4 * 2 + (size_t)kWarps * 16 * d * 4;
  if (OnePassLayout(d, group, split_keys).tm < merge) return 0;
  // four CTAs per SM (the occupancy it was measured at; with fewer, more of
  // each CTA's per-chunk latency shows)
  return bytes <= 56 * 1024 ? bytes : 0;
}

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream) {
  if (p.batch == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128>(p, kmap, vmap, stream) : launch_d<64>(p, kmap, vmap, stream);
}

}  // namespace attn
