// backward.cu -- varlen GQA attention backward on tcgen05 (sm_100a).
//
// NVIDIA/Model-Optimizer PR 1034 ("Add Triton unified attention kernel with
// HuggingFace integration"): the kernel serves training through autograd, so
// its masked softmax(Q K^T * scale) V needs dQ, dK and dV.  From the forward's
// output O and log-sum-exp L (natural log), with dO the output gradient:
//   P = exp(scale * Q K^T - L)            (recomputed tile by tile, masked)
//   Delta_i = <dO_i, O_i>                 (= sum_j P_ij dP_ij)
//   dP = dO V^T,  dS = P * (dP - Delta)
//   dV = P^T dO,  dK = scale * dS^T Q,  dQ = scale * dS K
// summed over the q-heads of each GQA group for dK and dV.
//
// Three kernels, no atomics (the result is deterministic):
//   bwd_delta_kernel: Delta per (query, q-head), one warp per row;
//   bwd_dkdv_kernel:  one CTA per (128-key tile, kv-head, sequence); it keeps
//       its K and V tiles in shared memory and dK, dV in TMEM while it walks
//       the 128-row query blocks of every q-head of the group that see the
//       tile: S^T = K Q^T and dP^T = V dO^T on tcgen05, P^T and dS^T by two
//       elementwise warpgroups (thread = key, each half of the block's
//       queries), then dV += P^T dO and dK += dS^T Q with P^T, dS^T read from
//       TMEM;
//   bwd_dq_kernel:    one CTA per (128-row query block, q-head, sequence); it
//       walks the key tiles the block sees: S = Q K^T, dP = dO V^T, dS by the
//       elementwise warpgroups (thread = query, each half of the tile's keys),
//       dQ += dS K with dS read from TMEM.
// S and dP are computed twice (once per kernel): two more tensor-core passes
// than a single kernel that adds dQ with atomics, no atomic traffic.
// TMEM (512 columns): dK/dV kernel S^T [0,128) -> P^T, dP^T [128,256) ->
// dS^T, dV [256,256+d), dK [384,384+d); dQ kernel S [0,128), dP [128,256)
// -> dS, dQ [256,256+d).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace attn {
namespace {

constexpr int BT = 128;                      // keys per tile, queries per block
constexpr int kQStages = 2;                  // dK/dV kernel: query blocks in flight
constexpr int kKVStages = 2;                 // dQ kernel: key tiles in flight
constexpr int kEwWarps = 16;                 // four elementwise warpgroups, 32 columns each
constexpr int kProducerWarp = kEwWarps;
constexpr int kMmaWarp = kEwWarps + 1;
constexpr int kThreads = 32 * (kEwWarps + 2);
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 1000000000ull;

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

ATTN_DEVICE void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
      : "memory");
}

// Bounded wait shared by all roles: gives up after one second (or when
// another role gave up), raising the timeout bit.
ATTN_DEVICE bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag, unsigned int *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, 20000)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  *abort_flag = 1;
  raise_error(err, ATTN_DEVERR_TIMEOUT);
  return false;
}

// Wait (at most one second, no error) for the phase: used before the TMEM is
// released so that no MMA still runs.
ATTN_DEVICE void drain_bar(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait_sleep(bar, parity, 20000) || globaltimer_ns() - t0 > kWaitNs) return;
}

struct Seq {
  int q0, k0, s_q, s_k;
  bool bad;
};

ATTN_DEVICE Seq seq_at(const BwdParams &p, int b) {
  Seq s;
  s.q0 = __ldg(p.cu_q + b);
  const int q1 = __ldg(p.cu_q + b + 1);
  s.k0 = __ldg(p.cu_k + b);
  const int k1 = __ldg(p.cu_k + b + 1);
  s.s_q = q1 - s.q0;
  s.s_k = k1 - s.k0;
  s.bad = (s.q0 < 0) | (s.s_q < 0) | (q1 > p.total_q) | (s.s_q > p.max_q) | (s.k0 < 0) | (s.s_k < 0) |
          (k1 > p.total_k) | (s.s_k > p.max_k);
  return s;
}

// Query blocks [r0, r1) of a sequence that see key tile t.
ATTN_DEVICE void blocks_seeing(const BwdParams &p, const Seq &s, int t, int &r0, int &r1) {
  r1 = (s.s_q + BT - 1) / BT;
  r0 = 0;
  if (p.causal) {
    const int first = t * BT - (s.s_k - s.s_q);   // first query that sees the tile's first key
    r0 = first <= 0 ? 0 : min(r1, first / BT);
  }
}

// Key tiles [0, n) a query block sees.
ATTN_DEVICE int tiles_seen(const BwdParams &p, const Seq &s, int r) {
  const int i_last = min(s.s_q, (r + 1) * BT) - 1;
  const int k_end = p.causal ? min(s.s_k, i_last + (s.s_k - s.s_q) + 1) : s.s_k;
  return k_end > 0 ? (k_end + BT - 1) / BT : 0;
}

// K-major operand of 128 rows x D (D / 64 swizzled halves of 128-byte rows):
// descriptor offset of the kk-th 16-element step along D.
template <int D>
ATTN_DEVICE uint32_t kmajor_step(int kk) {
  return (uint32_t)(((kk >> 2) * (BT * 128) + (kk & 3) * 32) >> 4);
}


// ---------------------------------------------------------------------------
// Delta_i = <dO_i, O_i>, one warp per (query, q-head) row
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(BwdParams p) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.total_q * p.h_q;
  const long long stride = (long long)gridDim.x * 8;
  for (long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); row < rows; row += stride) {
    const uint16_t *o = p.out + row * D + lane * E;
    const uint16_t *g = p.dout + row * D + lane * E;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const uint32_t ov = *reinterpret_cast<const uint32_t *>(o + e);
      const uint32_t gv = *reinterpret_cast<const uint32_t *>(g + e);
      acc = fmaf(bf16_lo(ov), bf16_lo(gv), acc);
      acc = fmaf(bf16_hi(ov), bf16_hi(gv), acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) p.delta[row] = acc;
  }
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <int D>
struct KvLayout {
  static constexpr int kTile = BT * D * 2;             // 128 rows x D bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;                 // [stage] query block
  static constexpr int kDO = kQ + kQStages * kTile;     // [stage] its output gradient
  static constexpr int kVec = kDO + kQStages * kTile;   // [stage] L * log2(e) [128], Delta [128]
  static constexpr int kBar = kVec + kQStages * BT * 2 * 4;
  // kv_full, q_full[S], q_empty[S], s_full, dp_full, p_done, ds_done, done
  static constexpr int kNumBars = 6 + 2 * kQStages;
  static constexpr int kMisc = kBar + kNumBars * 8;     // TMEM address, abort flag
  // at least ~116 KB, so that one CTA (and its 512 TMEM columns) owns an SM
  static constexpr int kBytes = (kMisc + 16 + 1024 > 118 * 1024) ? kMisc + 16 + 1024 : 118 * 1024;
  static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap dmap,
                    BwdParams p) {
  using L = KvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint64_t *kv_full = bars, *q_full = bars + 1, *q_empty = q_full + kQStages;
  uint64_t *s_full = q_empty + kQStages, *dp_full = s_full + 1, *p_done = dp_full + 1, *ds_done = p_done + 1;
  uint64_t *done = ds_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kMisc + 4);
  float *vec = reinterpret_cast<float *>(sm + L::kVec);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the key tiles of one (sequence, kv-head) are neighbours in launch order,
  // so they run together and read its query blocks while those sit in L2
  const int t = (int)(blockIdx.x % (unsigned)p.kt_max);
  const int grp = (int)(blockIdx.x / (unsigned)p.kt_max);
  const int hk = grp % p.h_kv, b = grp / p.h_kv;
  const int G = p.group;
  const Seq s = seq_at(p, b);
  if (s.bad || t * BT >= s.s_k) return;       // the whole CTA leaves before any barrier
  int r0, r1;
  blocks_seeing(p, s, t, r0, r1);
  const int per_head = r1 - r0;
  const int nb = G * per_head;                 // query blocks to visit: (q-head g, block r0 + i)

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int st = 0; st < kQStages; ++st) {
      mbar_init(&q_full[st], 1);
      mbar_init(&q_empty[st], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_done, kEwWarps);
    mbar_init(ds_done, kEwWarps);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);

  if (warp == kProducerWarp) {
    // ---------------- TMA producer (the whole warp; lane 0 issues) ----------------
    if (nb > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&qmap);
        tma_prefetch_desc(&dmap);
        mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sm + L::kK + h * BT * 128, &kmap, kv_full, h * 64, hk, s.k0 + t * BT);
          tma_load_3d(sm + L::kV + h * BT * 128, &vmap, kv_full, h * 64, hk, s.k0 + t * BT);
        }
      }
      int issued = 0;
      bool ok = true;
      for (int it = 0; it < nb && ok; ++it) {
        const int st = it % kQStages;
        if (it >= kQStages)
          ok = __all_sync(0xffffffffu, wait_bar(&q_empty[st], ((it / kQStages) - 1) & 1, abort_flag, p.err));
        if (!ok) break;
        const int hq = hk * G + it / per_head, r = r0 + it % per_head;
        float *lv = vec + st * 2 * BT;
        for (int m = lane; m < BT; m += 32) {
          const int i = r * BT + m;
          const bool in = i < s.s_q;
          const size_t row = (size_t)(s.q0 + (in ? i : 0)) * p.h_q + hq;
          lv[m] = in ? __ldg(p.lse + row) * kLog2e : 0.f;
          lv[BT + m] = in ? __ldg(p.delta + row) : 0.f;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[st], 2 * L::kTile);
          for (int h = 0; h < D / 64; ++h) {
            tma_load_3d(sm + L::kQ + st * L::kTile + h * BT * 128, &qmap, &q_full[st], h * 64, hq,
                        s.q0 + r * BT);
            tma_load_3d(sm + L::kDO + st * L::kTile + h * BT * 128, &dmap, &q_full[st], h * 64, hq,
                        s.q0 + r * BT);
          }
        }
        __syncwarp();
        issued = it + 1;
      }
      // a copy still in flight must land before the CTA's shared memory goes away
      if (!ok && lane == 0)
        for (int x = max(0, issued - kQStages); x < issued; ++x)
          wait_bar(&q_full[x % kQStages], (x / kQStages) & 1, abort_flag, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (the whole warp; one elected lane issues) ----------------
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(BT, BT, false);
    constexpr uint32_t idPV = idesc_bf16_f32(BT, D, true);
    bool ok = nb > 0 && __all_sync(0xffffffffu, wait_bar(kv_full, 0, abort_flag, p.err));
    const uint64_t dK0 = smem_desc_sw128(sbase + L::kK, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + L::kV, 16, 1024);
    for (int it = 0; it < nb && ok; ++it) {
      const int st = it % kQStages;
      ok = __all_sync(0xffffffffu, wait_bar(&q_full[st], (it / kQStages) & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const uint32_t sQ = sbase + L::kQ + st * L::kTile, sDO = sbase + L::kDO + st * L::kTile;
      if (leader) {
        const uint64_t dQ = smem_desc_sw128(sQ, 16, 1024), dDO = smem_desc_sw128(sDO, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem, dK0 + kmajor_step<D>(kk), dQ + kmajor_step<D>(kk), idS, kk > 0 ? 1u : 0u);
        tc_commit(s_full);     // the elementwise warps start on P^T while dP^T runs
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128, dV0 + kmajor_step<D>(kk), dDO + kmajor_step<D>(kk), idS, kk > 0 ? 1u : 0u);
        tc_commit(dp_full);
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, wait_bar(p_done, it & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      // B operands MN-major: rows = queries (K), 64-column halves of D (N)
      const uint64_t bDO = smem_desc_sw128(sDO, BT * 128, 1024), bQ = smem_desc_sw128(sQ, BT * 128, 1024);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {   // dV while the elementwise warps form dS^T
          const uint32_t a = 32 * (kk >> 1) + 8 * (kk & 1);    // P^T of queries [16 kk, 16 kk + 16)
          mma_ts(tmem + 256, tmem + a, bDO + ((kk * 16 * 128) >> 4), idPV, (it > 0 || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, wait_bar(ds_done, it & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          const uint32_t a = 128 + 32 * (kk >> 1) + 8 * (kk & 1);   // dS^T
          mma_ts(tmem + 384, tmem + a, bQ + ((kk * 16 * 128) >> 4), idPV, (it > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&q_empty[st]);
      }
      __syncwarp();
    }
    if (leader) tc_commit(done);   // every MMA issued so far is complete
    __syncwarp();
    drain_bar(done, 0);   // the TMEM is released only once no MMA runs
  } else {
    // ---------------- elementwise warpgroups: thread = key of the tile ----------------
    const int wg = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane, j = t * BT + row;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr, tP = tmem + lane_addr + 128;
    bool ok = true;
    for (int it = 0; it < nb && ok; ++it) {
      const int st = it % kQStages;
      ok = __all_sync(0xffffffffu, wait_bar(&q_full[st], (it / kQStages) & 1, abort_flag, p.err) &&
                                       wait_bar(s_full, it & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const int r = r0 + it % per_head;
      const float *lv = vec + st * 2 * BT;
      // this key may be seen by the block's queries (columns) [lo, hi)
      const int hi = j < s.s_k ? min(BT, s.s_q - r * BT) : 0;
      const int lo = p.causal ? max(0, j - (s.s_k - s.s_q) - r * BT) : 0;
      const int c = wg;                               // 32 queries [32 c, 32 c + 32) of the block
      const bool full = __all_sync(0xffffffffu, lo <= 32 * c && hi >= 32 * c + 32);
      {
        // P^T (while the dP^T product runs), handed over for dV; then dS^T
        uint32_t sr[32], pk[16];
        float pv[32];
        tmem_ld32(tS + 32 * c, sr);
        tmem_wait_ld();
        tie(sr);
        const float4 *l4 = reinterpret_cast<const float4 *>(lv + 32 * c);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 lq = l4[e4];
          const float la[4] = {lq.x, lq.y, lq.z, lq.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = 4 * e4 + u, col = 32 * c + e;
            const float x = ex2(fmaf(__uint_as_float(sr[e]), p.scale_log2, -la[u]));
            pv[e] = (full || (col >= lo && col < hi)) ? x : 0.f;
          }
          pk[2 * e4] = pack_bf16x2(pv[4 * e4], pv[4 * e4 + 1]);
          pk[2 * e4 + 1] = pack_bf16x2(pv[4 * e4 + 2], pv[4 * e4 + 3]);
        }
        tmem_st16(tS + 32 * c, pk);                   // P^T over this warpgroup's own S^T columns
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_done);
        ok = __all_sync(0xffffffffu, wait_bar(dp_full, it & 1, abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        uint32_t dr[32], dk[16];
        tmem_ld32(tP + 32 * c, dr);
        tmem_wait_ld();
        tie(dr);
        const float4 *d4 = reinterpret_cast<const float4 *>(lv + BT + 32 * c);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 dq = d4[e4];
          const float da[4] = {dq.x, dq.y, dq.z, dq.w};
          float dv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) dv[u] = pv[4 * e4 + u] * (__uint_as_float(dr[4 * e4 + u]) - da[u]);
          dk[2 * e4] = pack_bf16x2(dv[0], dv[1]);
          dk[2 * e4 + 1] = pack_bf16x2(dv[2], dv[3]);
        }
        tmem_st16(tP + 32 * c, dk);                   // dS^T over its own dP^T columns
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_done);
    }
    // epilogue: this warpgroup's half of the D columns of dV and dK
    const bool have = nb > 0;
    if (have) {
      ok = __all_sync(0xffffffffu, wait_bar(done, 0, abort_flag, p.err));
      tc_fence_after();
    }
    {
      // every lane takes part in the TMEM loads (they are warp-wide); only the
      // tile's keys that belong to the sequence are stored
      const size_t out_row = ((size_t)(s.k0 + min(j, s.s_k - 1)) * p.h_kv + hk) * D;
#pragma unroll 1
      for (int c = wg; c < D / 32; c += 4) {   // 32-column chunks of dV and dK
        uint32_t v[32], kv[32];
        if (have && ok) {
          tmem_ld32(tmem + lane_addr + 256 + 32 * c, v);
          tmem_ld32(tmem + lane_addr + 384 + 32 * c, kv);
          tmem_wait_ld();
          tie(v);
          tie(kv);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = kv[e] = 0u;
        }
        uint4 *dvp = reinterpret_cast<uint4 *>(p.dv + out_row + 32 * c);
        uint4 *dkp = reinterpret_cast<uint4 *>(p.dk + out_row + 32 * c);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w, w2;
          w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]), __uint_as_float(v[8 * q4 + 1]));
          w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3]));
          w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5]));
          w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7]));
          const float sc = p.scale;
          w2.x = pack_bf16x2(sc * __uint_as_float(kv[8 * q4 + 0]), sc * __uint_as_float(kv[8 * q4 + 1]));
          w2.y = pack_bf16x2(sc * __uint_as_float(kv[8 * q4 + 2]), sc * __uint_as_float(kv[8 * q4 + 3]));
          w2.z = pack_bf16x2(sc * __uint_as_float(kv[8 * q4 + 4]), sc * __uint_as_float(kv[8 * q4 + 5]));
          w2.w = pack_bf16x2(sc * __uint_as_float(kv[8 * q4 + 6]), sc * __uint_as_float(kv[8 * q4 + 7]));
          if (j < s.s_k) {
            dvp[q4] = w;
            dkp[q4] = w2;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
template <int D>
struct QLayout {
  static constexpr int kTile = BT * D * 2;
  static constexpr int kQ = 0;                          // the query block
  static constexpr int kDO = kQ + kTile;                // its output gradient
  static constexpr int kK = kDO + kTile;                // [stage] key tile
  static constexpr int kV = kK + kKVStages * kTile;     // [stage] value tile
  static constexpr int kBar = kV + kKVStages * kTile;
  // q_full, kv_full[S], kv_empty[S], s_full, dp_full, ds_done, done
  static constexpr int kNumBars = 5 + 2 * kKVStages;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = (kMisc + 16 + 1024 > 118 * 1024) ? kMisc + 16 + 1024 : 118 * 1024;
  static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap dmap,
                  BwdParams p) {
  using L = QLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint64_t *q_full = bars, *kv_full = bars + 1, *kv_empty = kv_full + kKVStages;
  uint64_t *s_full = kv_empty + kKVStages, *dp_full = s_full + 1, *ds_done = dp_full + 1, *done = ds_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // (sequence, q-head) fastest; the heaviest (last) causal query blocks first
  const int bh = (int)(blockIdx.x % (unsigned)(p.batch * p.h_q));
  const int r = p.qb_max - 1 - (int)(blockIdx.x / (unsigned)(p.batch * p.h_q));
  const int hq = bh % p.h_q, b = bh / p.h_q;
  const int hk = hq / p.group;
  const Seq s = seq_at(p, b);
  if (s.bad) {
    if (threadIdx.x == 0 && r == p.qb_max - 1 && hq == 0) raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
    return;
  }
  if (r * BT >= s.s_q) return;
  const int nt = tiles_seen(p, s, r);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int st = 0; st < kKVStages; ++st) {
      mbar_init(&kv_full[st], 1);
      mbar_init(&kv_empty[st], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_done, kEwWarps);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(sm);

  if (warp == kProducerWarp) {
    // ---------------- TMA producer ----------------
    if (nt > 0) {
      bool ok = true;
      int issued = 0;
      if (lane == 0) {
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&vmap);
        mbar_arrive_expect_tx(q_full, 2 * L::kTile);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(sm + L::kQ + h * BT * 128, &qmap, q_full, h * 64, hq, s.q0 + r * BT);
          tma_load_3d(sm + L::kDO + h * BT * 128, &dmap, q_full, h * 64, hq, s.q0 + r * BT);
        }
      }
      for (int jt = 0; jt < nt && ok; ++jt) {
        const int st = jt % kKVStages;
        if (jt >= kKVStages)
          ok = __all_sync(0xffffffffu, wait_bar(&kv_empty[st], ((jt / kKVStages) - 1) & 1, abort_flag, p.err));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&kv_full[st], 2 * L::kTile);
          for (int h = 0; h < D / 64; ++h) {
            tma_load_3d(sm + L::kK + st * L::kTile + h * BT * 128, &kmap, &kv_full[st], h * 64, hk,
                        s.k0 + jt * BT);
            tma_load_3d(sm + L::kV + st * L::kTile + h * BT * 128, &vmap, &kv_full[st], h * 64, hk,
                        s.k0 + jt * BT);
          }
        }
        __syncwarp();
        issued = jt + 1;
      }
      if (lane == 0) {
        // copies still in flight must land before the CTA's shared memory goes away
        wait_bar(q_full, 0, abort_flag, nullptr);
        if (!ok)
          for (int x = max(0, issued - kKVStages); x < issued; ++x)
            wait_bar(&kv_full[x % kKVStages], (x / kKVStages) & 1, abort_flag, nullptr);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue ----------------
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(BT, BT, false);
    constexpr uint32_t idPV = idesc_bf16_f32(BT, D, true);
    bool ok = nt > 0 && __all_sync(0xffffffffu, wait_bar(q_full, 0, abort_flag, p.err));
    const uint64_t aQ = smem_desc_sw128(sbase + L::kQ, 16, 1024);
    const uint64_t aDO = smem_desc_sw128(sbase + L::kDO, 16, 1024);
    // S of tile jt into columns [0, 128), its dP into [128, 256)
    auto issue_s = [&](int jt) {
      if (leader) {
        const uint64_t bK = smem_desc_sw128(sbase + L::kK + (jt % kKVStages) * L::kTile, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem, aQ + kmajor_step<D>(kk), bK + kmajor_step<D>(kk), idS, kk > 0 ? 1u : 0u);
        tc_commit(s_full);
      }
      __syncwarp();
    };
    auto issue_dp = [&](int jt) {
      if (leader) {
        const uint64_t bV = smem_desc_sw128(sbase + L::kV + (jt % kKVStages) * L::kTile, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128, aDO + kmajor_step<D>(kk), bV + kmajor_step<D>(kk), idS, kk > 0 ? 1u : 0u);
        tc_commit(dp_full);
      }
      __syncwarp();
    };
    // Per tile: S, dP (the elementwise warps form P while dP runs); once dS
    // is written (over dP's columns) the next tile's S, then dQ, then the next
    // dP, so the next exponentials overlap dQ and dP.
    if (ok) ok = __all_sync(0xffffffffu, wait_bar(&kv_full[0], 0, abort_flag, p.err));
    if (ok) {
      tc_fence_after();
      issue_s(0);
      issue_dp(0);
    }
    for (int jt = 0; jt < nt && ok; ++jt) {
      const int st = jt % kKVStages;
      const uint32_t sK = sbase + L::kK + st * L::kTile;
      ok = __all_sync(0xffffffffu, wait_bar(ds_done, jt & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const bool more = jt + 1 < nt;
      if (more) {
        ok = __all_sync(0xffffffffu,
                        wait_bar(&kv_full[(jt + 1) % kKVStages], ((jt + 1) / kKVStages) & 1, abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        issue_s(jt + 1);
      }
      if (leader) {
        // B = the key tile MN-major: rows = keys (K), 64-column halves of D (N)
        const uint64_t bKmn = smem_desc_sw128(sK, BT * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          const uint32_t a = 128 + 32 * (kk >> 1) + 8 * (kk & 1);   // dS of keys [16 kk, 16 kk + 16)
          mma_ts(tmem + 256, tmem + a, bKmn + ((kk * 16 * 128) >> 4), idPV, (jt > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&kv_empty[st]);
      }
      __syncwarp();
      if (more) issue_dp(jt + 1);
    }
    if (leader) tc_commit(done);
    __syncwarp();
    drain_bar(done, 0);
  } else {
    // ---------------- elementwise warpgroups: thread = query of the block ----------------
    const int wg = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane, i = r * BT + row;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr, tP = tmem + lane_addr + 128;
    const bool in = i < s.s_q;
    const size_t vrow = (size_t)(s.q0 + (in ? i : 0)) * p.h_q + hq;
    const float lse2 = in ? __ldg(p.lse + vrow) * kLog2e : 0.f;
    const float delta = in ? __ldg(p.delta + vrow) : 0.f;
    // this query sees the keys [0, k_lim) of its sequence
    const int k_lim = in ? (p.causal ? min(s.s_k, i + (s.s_k - s.s_q) + 1) : s.s_k) : 0;
    bool ok = true;
    for (int jt = 0; jt < nt && ok; ++jt) {
      ok = __all_sync(0xffffffffu, wait_bar(s_full, jt & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const int lim = k_lim - jt * BT;                 // allowed columns of this tile: [0, lim)
      const int c = wg;                               // keys [32 c, 32 c + 32) of the tile
      const bool full = __all_sync(0xffffffffu, lim >= 32 * c + 32);
      {
        // P while the dP product runs, then dS
        uint32_t sr[32], dr[32], dk[16];
        float pv[32];
        tmem_ld32(tS + 32 * c, sr);
        tmem_wait_ld();
        tie(sr);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = ex2(fmaf(__uint_as_float(sr[e]), p.scale_log2, -lse2));
          pv[e] = (full || 32 * c + e < lim) ? x : 0.f;
        }
        ok = __all_sync(0xffffffffu, wait_bar(dp_full, jt & 1, abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        tmem_ld32(tP + 32 * c, dr);
        tmem_wait_ld();
        tie(dr);
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          dk[e / 2] = pack_bf16x2(pv[e] * (__uint_as_float(dr[e]) - delta),
                                  pv[e + 1] * (__uint_as_float(dr[e + 1]) - delta));
        tmem_st16(tP + 32 * c, dk);                   // dS over this warpgroup's own dP columns
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_done);
    }
    const bool have = nt > 0;
    if (have) {
      ok = __all_sync(0xffffffffu, wait_bar(done, 0, abort_flag, p.err));
      tc_fence_after();
    }
    {
      // warp-wide TMEM loads by every lane; rows of the sequence are stored
      const size_t out_row = ((size_t)(s.q0 + (in ? i : 0)) * p.h_q + hq) * D;
#pragma unroll 1
      for (int c = wg; c < D / 32; c += 4) {
        uint32_t v[32];
        if (have && ok) {
          tmem_ld32(tmem + lane_addr + 256 + 32 * c, v);
          tmem_wait_ld();
          tie(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        uint4 *dqp = reinterpret_cast<uint4 *>(p.dq + out_row + 32 * c);
        const float sc = p.scale;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(sc * __uint_as_float(v[8 * q4 + 0]), sc * __uint_as_float(v[8 * q4 + 1]));
          w.y = pack_bf16x2(sc * __uint_as_float(v[8 * q4 + 2]), sc * __uint_as_float(v[8 * q4 + 3]));
          w.z = pack_bf16x2(sc * __uint_as_float(v[8 * q4 + 4]), sc * __uint_as_float(v[8 * q4 + 5]));
          w.w = pack_bf16x2(sc * __uint_as_float(v[8 * q4 + 6]), sc * __uint_as_float(v[8 * q4 + 7]));
          if (in) dqp[q4] = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
cudaError_t launch_bwd_d(const BwdParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                         const CUtensorMap &vmap, const CUtensorMap &dmap, cudaStream_t stream) {
  const long long rows = (long long)p.total_q * p.h_q;
  if (rows > 0) {
    const long long want = (rows + 7) / 8, cap = (long long)num_sms() * 8;
    bwd_delta_kernel<D><<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(p);
  }
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       KvLayout<D>::kBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, QLayout<D>::kBytes);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<(unsigned)p.kt_max * p.batch * p.h_kv, kThreads, KvLayout<D>::kBytes, stream>>>(
      qmap, kmap, vmap, dmap, p);
  bwd_dq_kernel<D><<<(unsigned)p.batch * p.h_q * p.qb_max, kThreads, QLayout<D>::kBytes, stream>>>(
      qmap, kmap, vmap, dmap, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                            const CUtensorMap &vmap, const CUtensorMap &dmap, cudaStream_t stream) {
  if (p.batch == 0 || p.qb_max == 0) return cudaSuccess;
  return p.d == 128 ? launch_bwd_d<128>(p, qmap, kmap, vmap, dmap, stream)
                    : launch_bwd_d<64>(p, qmap, kmap, vmap, dmap, stream);
}

}  // namespace attn
