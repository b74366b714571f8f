// prefill.cu -- varlen GQA attention forward on 5th-generation tensor cores.
//
// NVIDIA/Model-Optimizer PR 1034 ("Add Triton unified attention kernel with
// HuggingFace integration"): flash attention over packed variable-length
// batches, GQA, causal or non-causal.  NVIDIA/TensorRT-LLM PR 9821 ("Skip
// Softmax Attention"): the optional skip-softmax tile rule in the prefill.
//
// One CTA = one (q-head, 128-row q-block of one sequence).  Warp roles:
//   warp 0     TMA producer: Q tile once, then K_j / V_j tiles (128 keys x d)
//              into a 2-stage ring, 128-byte swizzled (3-D tensor maps over
//              the packed [tokens, heads, d] tensors; the GQA kv-head is a
//              tensor-map coordinate).
//   warp 1     TMEM allocation and the single-thread MMA issuer:
//              S_j = Q K_j^T  (tcgen05.mma kind::f16, A and B from shared
//              memory, fp32 accumulator in TMEM, two S buffers ping-pong),
//              O  += P_j V_j  (A = P_j read from TMEM where the softmax wrote
//              it over S_j, B = V_j from shared memory, MN-major).
//   warps 2-5  softmax warpgroup, one thread per query row (TMEM lane):
//              tcgen05.ld of S_j, varlen / causal masking, running max,
//              skip-softmax vote per 32-key sub-tile, p = 2^(s*scale*log2e - m),
//              row sums, P -> bf16 -> tcgen05.st, lazy O rescale (only when
//              the max grew by more than 2^8), epilogue O / l and LSE.
// TMEM columns: S buffer 0 [0,128), S buffer 1 [128,256), O [256, 256 + d).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace attn {
namespace {

constexpr int BM = kPrefillBlockM;
constexpr int BN = kPrefillBlockN;
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kDrainSpins = 1u << 20;

template <int D>
struct Smem {
  static constexpr int kTile = BM * D * 2;              // bytes of a 128 x D bf16 tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  // q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_done
  static constexpr int kNumBars = 1 + 3 * kStages + 2 + 2 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kUsed = kMisc + 64;
  // at least ~116 KB so that a single CTA (and its 512 TMEM columns) owns an SM
  static constexpr int kBytes = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
};

ATTN_DEVICE uint8_t *align1024(uint8_t *p) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Keep the compiler from using TMEM-load results before tcgen05.wait::ld.
ATTN_DEVICE void tie(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                 "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
                 "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
                 "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
                 "+r"(r[31]));
}

// Bounded wait that also gives up when another role raised the abort flag.
ATTN_DEVICE bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                               unsigned int *err) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  raise_error(err, ATTN_DEVERR_TIMEOUT);
  return false;
}

ATTN_DEVICE void drain(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kDrainSpins; ++i)
    if (mbar_try_wait(bar, parity)) return;
}

template <int D, bool SKIP>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, PrefillParams p) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *k_full = q_full + 1;
  uint64_t *v_full = k_full + kStages;
  uint64_t *kv_empty = v_full + kStages;
  uint64_t *s_full = kv_empty + kStages;
  uint64_t *p_full = s_full + 2;
  uint64_t *o_done = p_full + 2;
  uint32_t *misc = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  uint32_t *tmem_slot = misc;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  volatile uint32_t *skip_pv = misc + 2;        // [2]
  volatile uint32_t *votes = misc + 4;          // [2][4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hq = blockIdx.x;
  const int r = p.qb_max - 1 - (int)blockIdx.y / p.batch;   // heaviest q-blocks first
  const int b = (int)blockIdx.y % p.batch;

  // ---------------- sequence geometry ----------------
  const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
  const int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
  const int s_q = q1 - q0, s_k = k1 - k0;
  const bool bad = (q0 < 0) | (s_q < 0) | (q1 > p.total_q) | (s_q > p.max_q) | (k0 < 0) | (s_k < 0) |
                   (k1 > p.total_k) | (s_k > p.max_k);
  if (bad) {
    if (threadIdx.x == 0) raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
    return;
  }
  const int r0 = r * BM;
  if (r0 >= s_q) return;                       // block beyond this sequence
  const int i_last = min(r0 + BM, s_q) - 1;
  const int diag = s_k - s_q;                  // bottom-right causal alignment
  const int k_end = p.causal ? min(s_k, i_last + diag + 1) : s_k;      // keys any row may see
  const int n = k_end > 0 ? (k_end + BN - 1) / BN : 0;
  const int full_vis = p.causal ? min(s_k, r0 + diag + 1) : s_k;       // keys every row may see
  const int hk = hq / p.group;

  const uint32_t sQ = smem_u32(sm + L::kQ);
  const uint32_t sK = smem_u32(sm + L::kK);
  const uint32_t sV = smem_u32(sm + L::kV);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(o_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // =============== TMA producer ===============
    if (lane == 0 && n > 0) {
      const uint64_t keep = policy_evict_last();     // K/V tiles are re-read by the group's q-heads
      mbar_arrive_expect_tx(q_full, BM * D * 2);
      for (int h = 0; h < D / 64; ++h)
        tma_load_3d(sm + L::kQ + h * BM * 128, &qmap, q_full, h * 64, hq, q0 + r0);
      int j = 0;
      for (; j < n; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !wait_or_abort(&kv_empty[s], ((j / kStages) - 1) & 1, abort_flag, p.err))
          break;
        mbar_arrive_expect_tx(&k_full[s], BN * D * 2);
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d_hint(sm + L::kK + s * L::kTile + h * BN * 128, &kmap, &k_full[s], h * 64, hk,
                           k0 + j * BN, keep);
        mbar_arrive_expect_tx(&v_full[s], BN * D * 2);
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d_hint(sm + L::kV + s * L::kTile + h * BN * 128, &vmap, &v_full[s], h * 64, hk,
                           k0 + j * BN, keep);
      }
      if (*abort_flag) {
        // let copies still in flight land before the CTA's shared memory is released
        drain(q_full, 0);
        for (int x = max(0, j - kStages); x < j; ++x) {
          drain(&k_full[x % kStages], (x / kStages) & 1);
          drain(&v_full[x % kStages], (x / kStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // =============== MMA issuer ===============
    if (lane == 0 && n > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO = tmem + 256;
      bool ok = wait_or_abort(q_full, 0, abort_flag, p.err);
      auto issue_s = [&](int j) -> bool {
        const int s = j % kStages;
        if (!wait_or_abort(&k_full[s], (j / kStages) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(sQ + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + s * L::kTile + off, 16, 1024);
          mma_ss(tS[j & 1], a, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      uint32_t pv_started = 0;
      int issued = 0;
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !issue_s(j + 1)) break;
        if (!wait_or_abort(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const bool skip = SKIP && skip_pv[j & 1];
        if (!skip) {
          const int s = j % kStages;
          if (!wait_or_abort(&v_full[s], (j / kStages) & 1, abort_flag, p.err)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(sV + s * L::kTile + kk * 16 * 128, BN * 128, 1024);
            mma_ts(tO, tS[j & 1] + kk * 8, bd, idPV, (kk > 0 || pv_started) ? 1u : 0u);
          }
          pv_started = 1;
        }
        tc_commit(o_done);
        tc_commit(&kv_empty[j % kStages]);
        issued = j + 1;
      }
      if (*abort_flag && issued > 0) drain(o_done, (issued - 1) & 1);
    }
  } else {
    // =============== softmax warpgroup ===============
    const int quad = warp & 3;                    // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const int i = r0 + row;                       // query index inside the sequence
    const bool row_valid = i < s_q;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_true = -INFINITY;                     // running max (log2 units), drives the skip test
    float m_used = -INFINITY;                     // max the exponentials are taken against
    float l = 0.f;
    bool pv_any = false;                          // an earlier tile's PV was issued
    unsigned long long n_vis = 0, n_skip = 0;
    bool alive = true;

    for (int j = 0; j < n; ++j) {
      // a failed wait anywhere turns the rest of the loop into barrier-only
      // iterations, so the warps never disagree about the named barrier below
      bool ok = alive && wait_or_abort(&s_full[j & 1], (j >> 1) & 1, abort_flag, p.err);
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t tS = tmem + lane_addr + (j & 1) * 128;
      float s[128];
      if (ok) {
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) tie(sr[c]);
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = -INFINITY;
      }

      const int kbase = j * BN;
      if (kbase + BN > full_vis) {               // tile holds masked entries for some row
        const int lim = min(s_k, p.causal ? i + diag + 1 : s_k) - kbase;   // keys < lim allowed
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }

      bool pv_skip = false;
      if (SKIP) {
        // per 32-key sub-tile: vote skip when exp(tile max - running max) < threshold
        uint32_t my_votes = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float tmx = s[u * 32];
#pragma unroll
          for (int c = 1; c < 32; ++c) tmx = fmaxf(tmx, s[u * 32 + c]);
          const float t2 = tmx * sl2;
          const bool vote = !row_valid || (t2 == -INFINITY) || (t2 - m_true < p.thr_log2);
          m_true = fmaxf(m_true, t2);
          my_votes |= uint32_t(vote) << u;
        }
        uint32_t wv = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) wv |= uint32_t(__all_sync(0xffffffffu, (my_votes >> u) & 1u)) << u;
        if (lane == 0) votes[(j & 1) * 4 + quad] = wv | (ok ? 0u : 16u);
        named_bar_sync(1, 128);
        const uint32_t v0 = votes[(j & 1) * 4 + 0], v1 = votes[(j & 1) * 4 + 1];
        const uint32_t v2 = votes[(j & 1) * 4 + 2], v3 = votes[(j & 1) * 4 + 3];
        if ((v0 | v1 | v2 | v3) & 16u) {
          alive = false;
          continue;
        }
        uint32_t skip_bits = v0 & v1 & v2 & v3 & 15u;
        uint32_t vis_bits = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) vis_bits |= uint32_t(kbase + 32 * u < k_end) << u;
        skip_bits &= vis_bits;
        pv_skip = ((skip_bits | ~vis_bits) & 15u) == 15u;
        if (warp == 2 && lane == 0) {
          n_vis += __popc(vis_bits);
          n_skip += __popc(skip_bits);
          if (p.skip_mask && skip_bits) {
            for (int u = 0; u < 4; ++u) {
              if ((skip_bits >> u) & 1u) {
                const long long unit =
                    (((long long)b * p.qb_max + r) * p.h_q + hq) * p.kt_max + (kbase / 32 + u);
                atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
              }
            }
          }
          skip_pv[j & 1] = pv_skip ? 1u : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((skip_bits >> u) & 1u) {
#pragma unroll
            for (int c = 0; c < 32; ++c) s[u * 32 + c] = -INFINITY;
          }
      } else {
        if (!ok) {
          alive = false;
          break;
        }
        float tmx = s[0];
#pragma unroll
        for (int c = 1; c < 128; ++c) tmx = fmaxf(tmx, s[c]);
        m_true = fmaxf(m_true, tmx * sl2);
      }

      // lazy rescale: move the reference max only when it grew by more than 2^8
      float alpha = 1.f;
      if (m_true > m_used + kRescaleLog2 || (m_used == -INFINITY && m_true > -INFINITY)) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_true);
        m_used = m_true;
      }
      const float mref = (m_used == -INFINITY) ? 0.f : m_used;
      float rs = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2(fmaf(s[2 * c], sl2, -mref));
        const float p1 = ex2(fmaf(s[2 * c + 1], sl2, -mref));
        rs += p0 + p1;
        pk[c >> 5][c & 31] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;
      tmem_st32(tS, pk[0]);
      tmem_st32(tS + 32, pk[1]);
      tmem_wait_st();

      // rescale the O accumulator rows whose reference max moved
      if (pv_any && __any_sync(0xffffffffu, alpha != 1.f)) {
        const bool okw = __all_sync(0xffffffffu, wait_or_abort(o_done, (j - 1) & 1, abort_flag, p.err));
        if (!okw) alive = false;
        if (okw) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + 256 + c * 32, o);
            tmem_wait_ld();
            tie(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem + lane_addr + 256 + c * 32, o);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
      if (!SKIP && !alive) break;
      pv_any = pv_any || !pv_skip;
    }

    // ---------------- epilogue ----------------
    if (alive && n > 0) alive = wait_or_abort(o_done, (n - 1) & 1, abort_flag, p.err);
    alive = __all_sync(0xffffffffu, alive);
    tc_fence_after();
    const float inv = (l > 0.f) ? 1.f / l : 0.f;
    uint16_t *orow = p.out + ((size_t)(q0 + i) * p.h_q + hq) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      if (alive && n > 0) {
        tmem_ld32(tmem + lane_addr + 256 + c * 32, o);
        tmem_wait_ld();
        tie(o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      if (row_valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
          dst[v] = w;
        }
      }
    }
    if (row_valid && p.lse)
      p.lse[(size_t)(q0 + i) * p.h_q + hq] = (l > 0.f) ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
    if (SKIP && warp == 2 && lane == 0 && p.skip_counts) {
      atomicAdd(p.skip_counts + 0, n_vis);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool SKIP>
cudaError_t launch_t(const PrefillParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                     const CUtensorMap &vmap, cudaStream_t stream) {
  const int smem = Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, SKIP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.h_q, p.batch * p.qb_max);
  prefill_kernel<D, SKIP><<<grid, kThreads, smem, stream>>>(qmap, kmap, vmap, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, cudaStream_t stream) {
  if (p.batch == 0 || p.qb_max == 0) return cudaSuccess;
  const bool skip = p.thr_log2 > -INFINITY;
  if (p.d == 128)
    return skip ? launch_t<128, true>(p, qmap, kmap, vmap, stream)
                : launch_t<128, false>(p, qmap, kmap, vmap, stream);
  return skip ? launch_t<64, true>(p, qmap, kmap, vmap, stream)
              : launch_t<64, false>(p, qmap, kmap, vmap, stream);
}

}  // namespace attn
