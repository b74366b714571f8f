// prefill.cu -- varlen GQA attention forward on 5th-generation tensor cores.
//
// NVIDIA/Model-Optimizer PR 1034 ("Add Triton unified attention kernel with
// HuggingFace integration"): flash attention over packed variable-length
// batches, GQA, causal or non-causal.  NVIDIA/TensorRT-LLM PR 9821 ("Skip
// Softmax Attention"): the optional skip-softmax tile rule in the prefill.
//
// Persistent kernel, one CTA per SM, walking a static list of work items
// ordered heaviest first.  A work item is two 128-row query tiles that share
// every K/V tile: when the GQA group is even, the same q-block of two q-heads
// of one group (identical key ranges); otherwise two consecutive q-blocks of
// one head.  Warp roles (384 threads):
//   warps 0-3, 4-7  softmax warpgroups, one per query tile, one thread per
//                   query row (= TMEM lane): tcgen05.ld of S, varlen / causal
//                   masks, running max, skip-softmax vote per 32-key sub-tile,
//                   p = 2^(s*scale*log2e - m), row sums, P -> bf16 ->
//                   tcgen05.st over S, lazy O rescale (only when a row's max
//                   grew by more than 2^8), epilogue O / l and LSE.
//   warp 8          TMA producer: both Q tiles per item, then K_j / V_j into a
//                   2-stage ring (3-D tensor maps over the packed [tokens,
//                   heads, d] tensors, 128-byte swizzle, GQA kv-head as a
//                   coordinate).
//   warp 9          TMEM owner and MMA issuer (the warp runs the loop, one
//                   elected lane issues).  Per K/V tile j: PV0_j, S0_{j+1},
//                   PV1_j, S1_{j+1}, so the tensor core works on one tile while
//                   the other tile's softmax runs; each P.V starts on keys
//                   [0, 64) as soon as the softmax has written their P.
//   warps 10-11     idle (they only complete the third warpgroup).
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Waiting warps sleep in mbarrier.try_wait instead of spinning: every SM
// sub-partition hosts two softmax warps, and spinning waiters took issue
// slots from the one computing exponentials.
#include <limits.h>
#include <math.h>

#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace attn {
namespace {

constexpr int BM = kPrefillBlockM;
constexpr int BN = kPrefillBlockN;
constexpr int kStages = 2;
constexpr int kNQ = 2;                         // query tiles per work item
constexpr int kProducerWarp = 4 * kNQ;
constexpr int kMmaWarp = kProducerWarp + 1;
constexpr int kSchedWarp = kMmaWarp + 1;
constexpr int kSchedDepth = 4;                 // work items claimed ahead
constexpr int kSchedConsumers = 4 * kNQ + 2;   // warps that read each claimed item
// Sequences ranked for the sequence-major item order (batches of up to
// kRankMax sequences; larger batches keep their own order).
constexpr int kRankMax = 32;
// Work-claim slots.  A slot's word is (launch tag << 32) | next claim number,
// 0 when free.  Every CTA of a launch first takes the slot for its launch's
// tag (compare-and-swap from 0, or finding the tag already there); a CTA that
// finds another launch's tag waits, bounded, until that launch frees it.
// Claims are plain atomic adds.  A launch makes exactly `items` claims (each
// CTA claims until it draws a number past the items), so the claim that draws
// items - 1 is its last and puts the word back to 0.  Launches take slots in
// turn; two that meet on a slot therefore run one after the other's claims
// instead of sharing a counter.
constexpr int kWorkSlots = 64;
__device__ unsigned long long g_work[kWorkSlots];
constexpr int kThreads = 384;                  // softmax warpgroups 0, 1; warpgroup 2: TMA, MMA, 2 idle
// Register split: launched at 168 per thread (384 x 168 = 64 512), the
// producer / MMA warpgroup gives back down to 120 and each softmax warpgroup
// grows to 192: 2 x 128 x 192 + 128 x 120 = 64 512 (no spills either side).
constexpr uint32_t kRegsSoftmax = 192;
constexpr uint32_t kRegsOther = 120;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kDrainSpins = 1u << 20;
constexpr uint32_t kSleepHintNs = 20000;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

template <int D>
struct Smem {
  static constexpr int kTile = BM * D * 2;              // bytes of a 128 x D bf16 tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kNQ * kTile;
  static constexpr int kV = kK + kStages * kTile;
  // output staging: per query tile, 64 columns x 128 rows of bf16 (one store box)
  static constexpr int kStageBytes = BM * 64 * 2;
  static constexpr int kStage = kV + kStages * kTile;
  static constexpr int kBar = kStage + kNQ * kStageBytes;
  // q_full, q_empty, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[NQ], p_full[NQ], o_done[NQ],
  // o_free[NQ], p_half[NQ], sched_full[SD], sched_empty[SD], votes_ready[NQ][2]
  static constexpr int kNumBars = 2 + 4 * kStages + 5 * kNQ + 2 * kSchedDepth + 2 * kNQ;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static_assert(kMisc % 16 == 0, "the vote words are read as 16-byte vectors");
  static constexpr int kUsed = kMisc + 128;
  // at least ~116 KB so that a single CTA (and its 512 TMEM columns) owns an SM
  static constexpr int kBytes = (kUsed + 1024 > 118 * 1024) ? kUsed + 1024 : 118 * 1024;
  static_assert(kBytes <= 227 * 1024, "shared memory per CTA");
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
  if (mbar_try_wait(bar, parity)) return true;
  // suspended waits, bounded both in time (one second) and in count
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait_sleep(bar, parity, kSleepHintNs)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
  *abort_flag = 1;
  raise_error(err, ATTN_DEVERR_TIMEOUT);
  return false;
}

// Take work-claim slot `slot` for the launch tagged `tag` (see g_work).  False
// (ATTN_DEVERR_BUSY raised) when another launch held it for longer than the
// wait limit.
ATTN_DEVICE bool acquire_slot(unsigned long long *slot, uint32_t tag, unsigned int *err) {
  const unsigned long long mine = (unsigned long long)tag << 32;
  uint64_t t0 = 0;
  for (;;) {
    const unsigned long long prev = atomicCAS(slot, 0ull, mine);
    if (prev == 0ull || (uint32_t)(prev >> 32) == tag) return true;
    const uint64_t now = globaltimer_ns();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > kWaitLimitNs) {
      raise_error(err, ATTN_DEVERR_BUSY);
      return false;
    }
    __nanosleep(1000);
  }
}

ATTN_DEVICE void drain(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kDrainSpins; ++i)
    if (mbar_try_wait(bar, parity)) return;
}

// ---------------------------------------------------------------------------
// work items and per-tile geometry
// ---------------------------------------------------------------------------
struct Item {
  int b;
  int hq[kNQ];
  int r[kNQ];
};

ATTN_DEVICE int num_items(const PrefillParams &p) {
  if (p.group % 2 == 0) return p.batch * p.qb_max * (p.h_q / 2);
  return p.batch * ((p.qb_max + 1) / 2) * p.h_q;
}

// With sequences outermost, batches of up to kRankMax sequences take them
// longest first (the ranking is made by each CTA's scheduler warp).
ATTN_DEVICE bool ranked(const PrefillParams &p) { return p.seq_major && p.batch <= kRankMax; }

// Items are numbered heaviest first.  With seq_major == 0 the query-block
// index (counted from the last block) is the outer digit, so every
// sequence's last, causally heaviest, blocks come first; with seq_major == 1
// the ranked sequence is the outer digit and the query block the next.  The
// two query tiles of an item are two heads of one kv-head (even group), or
// two query blocks of one head (odd group).
ATTN_DEVICE Item item_at(const PrefillParams &p, const int *perm, int idx) {
  Item it;
  const bool even = p.group % 2 == 0;
  const int n_in = even ? p.h_q / 2 : p.h_q;                   // items per (sequence, block step)
  const int n_rr = even ? p.qb_max : (p.qb_max + 1) / 2;       // block steps per sequence
  int bs, rr, h;
  if (p.seq_major) {
    const int per = n_rr * n_in;
    bs = idx / per;
    const int rem = idx - bs * per;
    rr = rem / n_in;
    h = rem - rr * n_in;
  } else {
    const int per = p.batch * n_in;
    rr = idx / per;
    const int rem = idx - rr * per;
    bs = rem / n_in;
    h = rem - bs * n_in;
  }
  it.b = ranked(p) ? perm[bs] : bs;
  if (even) {
    const int r = p.qb_max - 1 - rr;
    it.hq[0] = 2 * h;
    it.hq[1] = 2 * h + 1;
    it.r[0] = r;
    it.r[1] = r;
  } else {
    const int rp = n_rr - 1 - rr;
    it.hq[0] = h;
    it.hq[1] = h;
    it.r[0] = 2 * rp;
    it.r[1] = 2 * rp + 1;
  }
  return it;
}

struct Seq {
  int q0, k0, s_q, s_k;
  bool bad;
};

ATTN_DEVICE Seq seq_at(const PrefillParams &p, int b) {
  Seq s;
  s.q0 = __ldg(p.cu_q + b);
  const int q1 = __ldg(p.cu_q + b + 1);
  s.s_q = q1 - s.q0;
  s.bad = (s.q0 < 0) | (s.s_q < 0) | (q1 > p.total_q) | (s.s_q > p.max_q);
  if (p.paged) {
    s.k0 = 0;
    s.s_k = __ldg(p.seq_lens_k + b);
    s.bad |= (s.s_k < 0) | (s.s_k > p.max_k) | (s.s_k > p.max_pages * kPageSize);
  } else {
    s.k0 = __ldg(p.cu_k + b);
    const int k1 = __ldg(p.cu_k + b + 1);
    s.s_k = k1 - s.k0;
    s.bad |= (s.k0 < 0) | (s.s_k < 0) | (k1 > p.total_k) | (s.s_k > p.max_k);
  }
  return s;
}

struct TileGeo {
  int r0;         // first query row of the tile inside the sequence
  int n;          // K/V tiles the tile needs
  int k_end;      // keys any row of the tile may see
  int full_vis;   // keys every row of the tile may see
  bool active;    // the tile holds rows of the sequence
};

ATTN_DEVICE TileGeo tile_geo(const PrefillParams &p, const Seq &s, int r) {
  TileGeo g;
  g.r0 = r * BM;
  g.active = !s.bad && g.r0 < s.s_q;
  const int i_last = min(g.r0 + BM, s.s_q) - 1;
  const int diag = s.s_k - s.s_q;                          // bottom-right causal alignment
  g.k_end = p.causal ? min(s.s_k, i_last + diag + 1) : s.s_k;
  g.full_vis = p.causal ? min(s.s_k, g.r0 + diag + 1) : s.s_k;
  g.n = (g.active && g.k_end > 0) ? (g.k_end + BN - 1) / BN : 0;
  return g;
}

// ---------------------------------------------------------------------------
// softmax pieces
// ---------------------------------------------------------------------------
// AND of four consecutive 32-bit words in shared memory (16-byte aligned),
// read with one volatile vector load.
ATTN_DEVICE uint32_t and4_shared(const volatile uint32_t *p) {
  uint32_t a, b, c, d;
  asm volatile("ld.volatile.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(smem_u32(const_cast<const uint32_t *>(p))));
  return a & b & c & d;
}

// 16 columns of a warp's TMEM lanes from 16 consecutive registers.
ATTN_DEVICE void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
      : "memory");
}

// -inf for the columns at or beyond `lim` (keys the row may not see).
ATTN_DEVICE void mask_cols(uint32_t (&sr)[4][32], int lim) {
#pragma unroll
  for (int c = 0; c < 128; ++c)
    if (c >= lim) sr[c >> 5][c & 31] = 0xff800000u;
}

ATTN_DEVICE float fmax3u(float m, uint32_t a, uint32_t b) {
  return max3(m, __uint_as_float(a), __uint_as_float(b));
}

// Raw maxima of the four 32-column sub-tiles of a row (two chains each).
ATTN_DEVICE void max_sub4(const uint32_t (&sr)[4][32], float (&um)[4]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float a = -INFINITY, b = -INFINITY;
#pragma unroll
    for (int c = 0; c < 32; c += 4) {
      a = fmax3u(a, sr[u][c], sr[u][c + 1]);
      b = fmax3u(b, sr[u][c + 2], sr[u][c + 3]);
    }
    um[u] = fmaxf(a, b);
  }
}

// p = 2^(s * sl2 - mref) for 64 columns of a row (32-column chunks a, b),
// packed to bf16 pairs and stored to TMEM at `taddr` (32 columns, as two
// 16-column stores so that the first is under way while the rest is
// computed); the sums of p over chunk a and chunk b go to ps[0], ps[1].
ATTN_DEVICE void exp64_to_tmem(const uint32_t (&a)[32], const uint32_t (&b)[32], float sl2, float mref,
                               uint32_t taddr, float *ps) {
  const uint64_t scale2 = f2_pack(sl2, sl2), neg_m2 = f2_pack(-mref, -mref);
  uint64_t acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = f2_pack(0.f, 0.f);
  uint32_t pk[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int e = (2 * q) & 31;
    const uint32_t x0u = q < 16 ? a[e] : b[e], x1u = q < 16 ? a[e + 1] : b[e + 1];
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(x0u), __uint_as_float(x1u)), scale2, neg_m2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const float p0 = ex2(x0), p1 = ex2(x1);
    const int ac = (q < 16 ? 0 : 2) + (q & 1);
    acc[ac] = f2_add(acc[ac], f2_pack(p0, p1));
    pk[q] = pack_bf16x2(p0, p1);
    if (q == 15) tmem_st16(taddr, pk);
  }
  tmem_st16(taddr + 16, pk + 16);
  float x0, x1;
  f2_unpack(f2_add(acc[0], acc[1]), x0, x1);
  ps[0] = x0 + x1;
  f2_unpack(f2_add(acc[2], acc[3]), x0, x1);
  ps[1] = x0 + x1;
}

// p = 2^(s * sl2 - mref) for one 32-column sub-tile of a row, packed to bf16
// pairs and stored to TMEM at `taddr` (16 columns); returns the sum of p
// (the same pairing as exp64_to_tmem's per-chunk sums).
ATTN_DEVICE float exp32_to_tmem(const uint32_t (&a)[32], float sl2, float mref, uint32_t taddr) {
  const uint64_t scale2 = f2_pack(sl2, sl2), neg_m2 = f2_pack(-mref, -mref);
  uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
  uint32_t pk[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1])), scale2, neg_m2);
    float x0, x1;
    f2_unpack(x, x0, x1);
    const float p0 = ex2(x0), p1 = ex2(x1);
    acc[q & 1] = f2_add(acc[q & 1], f2_pack(p0, p1));
    pk[q] = pack_bf16x2(p0, p1);
  }
  tmem_st16(taddr, pk);
  float x0, x1;
  f2_unpack(f2_add(acc[0], acc[1]), x0, x1);
  return x0 + x1;
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int D, bool SKIP, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap omap,
                   PrefillParams p) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = align1024(smem_raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::kBar);
  uint64_t *q_full = bars;
  uint64_t *q_empty = q_full + 1;
  uint64_t *k_full = q_empty + 1;
  uint64_t *v_full = k_full + kStages;
  uint64_t *k_empty = v_full + kStages;         // [S] both tiles' S of the slot's K tile are done
  uint64_t *v_empty = k_empty + kStages;        // [S] both tiles' P.V of the slot's V tile are done
  uint64_t *s_full = v_empty + kStages;
  uint64_t *p_full = s_full + kNQ;
  uint64_t *o_done = p_full + kNQ;
  uint64_t *o_free = o_done + kNQ;
  uint64_t *p_half = o_free + kNQ;              // P of keys [0, 64) of the tile is in TMEM
  uint64_t *sched_full = p_half + kNQ;          // [kSchedDepth] a claimed item is in the ring
  uint64_t *sched_empty = sched_full + kSchedDepth;
  uint64_t *votes_ready = sched_empty + kSchedDepth;   // [kNQ][2] the four warps' votes are written
  uint32_t *misc = reinterpret_cast<uint32_t *>(sm + L::kMisc);
  uint32_t *tmem_slot = misc;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  // skip votes of the four warps of a softmax warpgroup, per query tile and
  // tile count mod 3: bit u = every row of the warp votes to skip 32-key
  // sub-tile u.  The warps read tile c's votes right after its votes_ready
  // phase and the MMA warp before it issues tile c's P.V; tile c + 3's votes
  // (the same slot) come after S of tile c + 3, which follows all of those.
  volatile uint32_t *votes = misc + 4;          // [kNQ][3][4]
  volatile int *ring = reinterpret_cast<volatile int *>(misc + 28);   // [kSchedDepth] claimed items
  // ranked sequences (written once, before the first claimed item is
  // published; a static array, so that its address takes no register)
  __shared__ int perm[kRankMax];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = num_items(p);
  // Work items are numbered heaviest first.  A CTA starts on item blockIdx.x
  // and then claims the next unclaimed one from the launch's counter (warp
  // kSchedWarp, kSchedDepth items ahead), so CTAs that drew light items take
  // more of them; the claimed item numbers reach every role through a ring in
  // shared memory.  -1 ends the work.
  auto pop_warp = [&](uint32_t n) -> int {      // whole-warp roles
    const uint32_t slot = n % kSchedDepth;
    const bool okw =
        __all_sync(0xffffffffu, wait_or_abort(&sched_full[slot], (n / kSchedDepth) & 1, abort_flag, p.err));
    const int idx = okw ? ring[slot] : -1;
    __syncwarp();
    if ((threadIdx.x & 31u) == 0u) mbar_arrive(&sched_empty[slot]);
    return idx;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < kNQ; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_free[t], 4);
      mbar_init(&p_half[t], 4);
      mbar_init(&votes_ready[2 * t], 4);
      mbar_init(&votes_ready[2 * t + 1], 4);
    }
    for (int q = 0; q < kSchedDepth; ++q) {
      mbar_init(&sched_full[q], 1);
      mbar_init(&sched_empty[q], kSchedConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    tma_prefetch_desc(&omap);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    regs_decrease<kRegsOther>();
  if (warp == kProducerWarp) {
    // =============== TMA producer ===============
    // The whole warp runs the loop; lane 0 issues the Q copies and the
    // contiguous K/V tiles.  With a paged cache a K/V tile is eight 16-token
    // pages, and lanes 0-7 each read one page number and issue that page's
    // boxes, so the many small copies do not queue behind one thread.
    {
      const uint64_t keep = policy_evict_last();     // K/V tiles are re-read by other q-heads
      uint32_t kv_c = 0, q_c = 0;
      uint32_t k_issued = 0, v_issued = 0;    // K / V tiles whose copies were issued
      bool ok = true;
      auto wait_all_p = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag, p.err));
      };
      for (uint32_t n = 0; ok; ++n) {
        const int idx = pop_warp(n);
        if (idx < 0) break;
        const Item it = item_at(p, perm, idx);
        const Seq sq = seq_at(p, it.b);
        if (sq.bad) continue;
        TileGeo g[kNQ];
        int nmax = 0;
#pragma unroll
        for (int t = 0; t < kNQ; ++t) {
          g[t] = tile_geo(p, sq, it.r[t]);
          nmax = max(nmax, g[t].n);
        }
        if (nmax == 0) continue;
        if (q_c > 0 && !(ok = wait_all_p(q_empty, (q_c - 1) & 1))) break;
        if (lane == 0) {
          int qbytes = 0;
          for (int t = 0; t < kNQ; ++t) qbytes += g[t].n > 0 ? BM * D * 2 : 0;
          mbar_arrive_expect_tx(q_full, qbytes);
          for (int t = 0; t < kNQ; ++t) {
            if (g[t].n == 0) continue;
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(sm + L::kQ + t * L::kTile + h * BM * 128, &qmap, q_full, h * 64, it.hq[t],
                          sq.q0 + g[t].r0);
          }
        }
        const int hk = it.hq[0] / p.group;
        const int32_t *bt = PAGED ? p.block_table + (size_t)it.b * p.max_pages : nullptr;
        // a paged tile's block-table entries are read one tile ahead, so that
        // their latency is not added to the copies' once a slot frees up
        auto page_raw = [&](int j) -> int {
          const int tok = j * BN + lane * kPageSize;
          return (PAGED && lane < BN / kPageSize && tok < sq.s_k) ? __ldg(bt + tok / kPageSize) : 0;
        };
        // K or V tile j of the item (global tile count c) into its ring slot,
        // once the slot's previous tile is no longer read
        auto load = [&](bool is_k, int j, uint32_t c, int raw) -> bool {
          const int s = c % kStages;
          uint64_t *full = is_k ? k_full : v_full;
          if (c >= kStages && !wait_all_p(is_k ? &k_empty[s] : &v_empty[s], ((c / kStages) - 1) & 1))
            return false;
          if (lane == 0) mbar_arrive_expect_tx(&full[s], BN * D * 2);
          __syncwarp();
          const CUtensorMap *map = is_k ? &kmap : &vmap;
          uint8_t *slot = sm + (is_k ? L::kK : L::kV) + s * L::kTile;
          if constexpr (!PAGED) {
            if (lane == 0)
              for (int h = 0; h < D / 64; ++h)
                tma_load_3d_hint(slot + h * BN * 128, map, &full[s], h * 64, hk, sq.k0 + j * BN, keep);
          } else if (lane < BN / kPageSize) {
            // one 16-token page per box; a page past the sequence (or a bad
            // block-table entry, reported) is read at a row beyond the cache,
            // which the copy fills with zeros
            const int tok = j * BN + lane * kPageSize;
            int page = p.num_pages;
            if (tok < sq.s_k) {
              page = raw;
              if (page < 0 || page >= p.num_pages) {
                if (is_k) raise_error(p.err, ATTN_DEVERR_BLOCK_TABLE);
                page = p.num_pages;
              }
            }
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d_hint(slot + lane * kPageSize * 128 + h * BN * 128, map, &full[s], h * 64, hk,
                               page * kPageSize, keep);
          }
          __syncwarp();
          return true;
        };
        // K runs one tile ahead of V: a K slot frees when both query tiles'
        // S of its tile are done, a V slot only when their P.V are, so the
        // next K tile (which the next S waits for) is fetched a tile earlier
        int raw0 = page_raw(0), raw1 = nmax > 1 ? page_raw(1) : 0;
        if (!(ok = load(true, 0, kv_c, raw0))) break;
        k_issued = kv_c + 1;
        for (int j = 0; j < nmax; ++j) {
          const int raw2 = j + 2 < nmax ? page_raw(j + 2) : 0;
          if (j + 1 < nmax) {
            if (!(ok = load(true, j + 1, kv_c + j + 1, raw1))) break;
            k_issued = kv_c + j + 2;
          }
          if (!(ok = load(false, j, kv_c + j, raw0))) break;
          v_issued = kv_c + j + 1;
          raw0 = raw1;
          raw1 = raw2;
        }
        if (!ok) break;
        kv_c += nmax;
        ++q_c;
      }
      if (!ok && lane == 0) {
        // let copies still in flight land before the CTA's shared memory is released
        if (q_c > 0) drain(q_full, (q_c - 1) & 1);
        for (uint32_t x = k_issued > kStages ? k_issued - kStages : 0; x < k_issued; ++x)
          drain(&k_full[x % kStages], (x / kStages) & 1);
        for (uint32_t x = v_issued > kStages ? v_issued - kStages : 0; x < v_issued; ++x)
          drain(&v_full[x % kStages], (x / kStages) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // =============== MMA issuer ===============
    // The whole warp runs the loop (waits, descriptor arithmetic) in
    // convergent code; one elected lane issues each MMA and commit.  The warp
    // shares its SM sub-partition with two busy softmax warps, so the
    // per-MMA instruction count matters: descriptors are built once per
    // group and stepped by constants (the 14-bit address field never
    // carries: shared addresses are below 2^18).
    const bool leader = elect_one();
    const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
    constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
    constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
    const uint32_t sQ = smem_u32(sm + L::kQ);
    const uint32_t sK = smem_u32(sm + L::kK);
    const uint32_t sV = smem_u32(sm + L::kV);
    uint32_t kv_c = 0, q_c = 0;
    uint32_t tile_c[kNQ] = {0, 0};   // tiles processed per query-tile slot (p_full / o_done phases)
    uint32_t item_c[kNQ] = {0, 0};   // items with work per slot (o_free phases)
    uint32_t vslot[kNQ] = {0, 0};    // tile_c mod 3: the slot of the tile's votes
    bool ok = true;
    auto wait_all = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag, p.err));
    };
    auto commit = [&](uint64_t *bar) {
      if (leader) tc_commit(bar);
      __syncwarp();
    };
    auto issue_s = [&](int t, uint32_t stage) {
      const uint64_t a0 = smem_desc_sw128(sQ + t * L::kTile, 16, 1024);
      const uint64_t b0 = smem_desc_sw128(sK + stage * L::kTile, 16, 1024);
      const uint32_t d = tmem + t * 128;
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
          mma_ss(d, a0 + off, b0 + off, idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[t]);
      }
      __syncwarp();
    };

    for (uint32_t n = 0; ok; ++n) {
      const int idx = pop_warp(n);
      if (idx < 0) break;
      const Item it = item_at(p, perm, idx);
      const Seq sq = seq_at(p, it.b);
      if (sq.bad) continue;
      TileGeo g[kNQ];
      int nmax = 0;
#pragma unroll
      for (int t = 0; t < kNQ; ++t) {
        g[t] = tile_geo(p, sq, it.r[t]);
        nmax = max(nmax, g[t].n);
      }
      if (nmax == 0) continue;
      if (!(ok = wait_all(q_full, q_c & 1))) break;
      if (!(ok = wait_all(&k_full[kv_c % kStages], (kv_c / kStages) & 1))) break;
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < kNQ; ++t)
        if (g[t].n > 0) issue_s(t, kv_c % kStages);
      commit(&k_empty[kv_c % kStages]);
      uint32_t pv_started[kNQ] = {0, 0};
      for (int j = 0; ok && j < nmax; ++j) {
        const uint32_t c = kv_c + j, st = c % kStages;
        bool v_ready = false, k_next_ready = false;
#pragma unroll
        for (int t = 0; t < kNQ; ++t) {
          if (!ok || j >= g[t].n) continue;
          ok = wait_all(&p_half[t], tile_c[t] & 1);
          if (ok && j == 0 && item_c[t] > 0) ok = wait_all(&o_free[t], (item_c[t] - 1) & 1);
          if (!ok) continue;
          tc_fence_after();
          // Skip-softmax: the four softmax warps' votes for this tile were
          // written before their P hand-off; a 32-key sub-tile is skipped when
          // every row votes for it, and its P.V MMAs (two 16-key steps) are not
          // issued (the softmax warps wrote no P for it and left it out of
          // their row sums; sub-tiles past the keys vote skip too).
          uint32_t skip_bits = 0;
          if constexpr (SKIP) skip_bits = and4_shared(votes + (t * 3 + vslot[t]) * 4);
          // With both sub-tiles of keys [64, 128) skipped the softmax warps
          // write nothing to this tile's TMEM after their first hand-off (S
          // is in their registers by then), so the next S is issued without
          // waiting for the second; with all four skipped, no P.V reads V.
          const bool hi_skip = SKIP && (skip_bits & 0xcu) == 0xcu;
          const bool all_skip = SKIP && (skip_bits & 0xfu) == 0xfu;
          if (!v_ready && !all_skip) {
            if (!(ok = wait_all(&v_full[st], (c / kStages) & 1))) continue;
            tc_fence_after();
            v_ready = true;
            if (PAGED && j == (sq.s_k - 1) / BN && (sq.s_k % kPageSize) != 0) {
              // the sequence's last page holds slots past its end (whatever the
              // cache has there); their p is 0, but 0 * NaN is not, so the V
              // rows are zeroed before the P.V MMAs read them
              const int r0 = sq.s_k - j * BN, r1 = (r0 + kPageSize - 1) / kPageSize * kPageSize;
              for (int x = lane; x < (r1 - r0) * (D / 64) * 8; x += 32) {
                const int h = x / ((r1 - r0) * 8), rem = x - h * (r1 - r0) * 8;
                const int r = r0 + rem / 8, ch = rem % 8;
                *reinterpret_cast<uint4 *>(sm + L::kV + st * L::kTile + h * BN * 128 + r * 128 + ch * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
          }
          const uint64_t v0 = smem_desc_sw128(sV + st * L::kTile, BN * 128, 1024);
          uint32_t acc = pv_started[t];
          const uint32_t d = tmem + 256 + t * 128, a = tmem + t * 128;
          // keys [0, 64) as soon as their P is written, the rest after
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < BN / 32; ++kk) {
              if ((skip_bits >> (kk / 2)) & 1u) continue;
              mma_ts(d, a + kk * 8, v0 + ((kk * 16 * 128) >> 4), idPV, acc);
              acc = 1u;
            }
          }
          __syncwarp();
          if (!hi_skip) {
            // (a skipped wait is safe: this p_full phase completes before the
            // next p_half one, which the next step waits for first)
            if (!(ok = wait_all(&p_full[t], tile_c[t] & 1))) continue;
            tc_fence_after();
            if (leader) {
#pragma unroll
              for (int kk = BN / 32; kk < BN / 16; ++kk) {
                if ((skip_bits >> (kk / 2)) & 1u) continue;
                mma_ts(d, a + kk * 8, v0 + ((kk * 16 * 128) >> 4), idPV, acc);
                acc = 1u;
              }
            }
          }
          pv_started[t] = __shfl_sync(0xffffffffu, acc, leader_lane);
          commit(&o_done[t]);
          ++tile_c[t];
          if constexpr (SKIP) vslot[t] = vslot[t] == 2 ? 0 : vslot[t] + 1;
          if (j + 1 < g[t].n) {
            if (!k_next_ready) {
              const uint32_t cn = c + 1;
              if (!(ok = wait_all(&k_full[cn % kStages], (cn / kStages) & 1))) continue;
              tc_fence_after();
              k_next_ready = true;
            }
            issue_s(t, (c + 1) % kStages);
          }
        }
        // the V slot is released only after its copy has landed, read or not
        if constexpr (SKIP) {
          if (ok && !v_ready) ok = wait_all(&v_full[st], (c / kStages) & 1);
        }
        if (ok) {
          // this tile's V, and the next tile's K once both S were issued above
          commit(&v_empty[st]);
          if (j + 1 < nmax) commit(&k_empty[(c + 1) % kStages]);
        }
      }
      if (!ok) break;
      commit(q_empty);
#pragma unroll
      for (int t = 0; t < kNQ; ++t) item_c[t] += g[t].n > 0 ? 1 : 0;
      kv_c += nmax;
      ++q_c;
    }
    // every MMA must be complete before the TMEM is released, and every
    // commit's arrival must have landed before the shared memory is
    if (leader) {
#pragma unroll
      for (int t = 0; t < kNQ; ++t)
        if (tile_c[t] > 0) drain(&o_done[t], (tile_c[t] - 1) & 1);
      if (kv_c > 0) {
        drain(&k_empty[(kv_c - 1) % kStages], ((kv_c - 1) / kStages) & 1);
        drain(&v_empty[(kv_c - 1) % kStages], ((kv_c - 1) / kStages) & 1);
      }
      if (q_c > 0) drain(q_empty, (q_c - 1) & 1);
    }
    __syncwarp();
  } else if (warp == kSchedWarp) {
    // =============== work claims ===============
    if (ranked(p)) {
      // rank the sequences by key length, longest first, ties in index
      // order, broken ones last; lane b holds sequence b, lane 0 writes the
      // ranking
      int key = INT_MIN;
      if (lane < p.batch) {
        const Seq sq = seq_at(p, lane);
        key = sq.bad ? INT_MIN + 1 : sq.s_k;
      }
      int rank = 0;
      for (int j = 0; j < p.batch; ++j) {
        const int kj = __shfl_sync(0xffffffffu, key, j);
        rank += (kj > key) || (kj == key && j < lane);
      }
      for (int r = 0; r < p.batch; ++r) {
        const unsigned int m = __ballot_sync(0xffffffffu, lane < p.batch && rank == r);
        if (lane == 0) perm[r] = __ffs(m) - 1;
      }
    }
    if (lane == 0) {
      unsigned long long *slot = &g_work[p.work_slot];
      const bool owned = acquire_slot(slot, p.work_tag, p.err);
      // the next claimed item number; the launch's last claim frees the slot
      auto claim = [&]() -> int {
        const unsigned long long old = atomicAdd(slot, 1ull);
        const uint32_t c = (uint32_t)old;
        if ((uint32_t)(old >> 32) != p.work_tag) raise_error(p.err, ATTN_DEVERR_BUSY);
        if (c + 1u == (uint32_t)items) atomicExch(slot, 0ull);
        return (int)gridDim.x + (int)c;
      };
      // an item holds work when one of its query tiles holds rows (a tile
      // whose rows see no key still writes zeros and -inf); items of a
      // sequence with broken cu_seqlens are reported and dropped here
      auto has_work = [&](int idx) {
        const Item it = item_at(p, perm, idx);
        const Seq sq = seq_at(p, it.b);
        if (sq.bad) {
          raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
          return false;
        }
        bool any = false;
#pragma unroll
        for (int t = 0; t < kNQ; ++t) any = any || tile_geo(p, sq, it.r[t]).active;
        return any;
      };
      // a CTA that could not take the slot does no work (the error is raised)
      int next = owned ? (int)blockIdx.x : items;
      for (uint32_t n = 0;; ++n) {
        while (next < items && !has_work(next)) next = claim();
        const uint32_t rs = n % kSchedDepth;
        if (n >= kSchedDepth &&
            !wait_or_abort(&sched_empty[rs], ((n / kSchedDepth) - 1) & 1, abort_flag, p.err))
          break;
        ring[rs] = next < items ? next : -1;
        mbar_arrive(&sched_full[rs]);
        if (next >= items) break;
        next = claim();
      }
      // after an abort, the remaining claims are still drawn, so that the
      // launch's count completes and the slot is freed
      while (owned && next < items) next = claim();
    }
  }
  } else {
    regs_increase<kRegsSoftmax>();
    // =============== softmax warpgroups ===============
    const int t = warp >> 2;                      // query tile of this warpgroup
    const int quad = warp & 3;                    // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + t * 128;
    const uint32_t tO = tmem + lane_addr + 256 + t * 128;
    const float sl2 = p.scale_log2;
    uint32_t tile_c = 0;
    bool alive = true;
    // skip-softmax counts of this warpgroup's units (kept by its first warp)
    unsigned long long n_vis = 0, n_skip = 0;

    for (uint32_t n = 0; alive; ++n) {
      const int idx = pop_warp(n);
      if (idx < 0) break;
      const Item it = item_at(p, perm, idx);
      const Seq sq = seq_at(p, it.b);
      const TileGeo g = tile_geo(p, sq, it.r[t]);
      if (!g.active) continue;
      const int hq = it.hq[t];
      const int i = g.r0 + row;                   // query index inside the sequence
      const bool row_valid = i < sq.s_q;
      const int diag = sq.s_k - sq.s_q;
      const int lim_row = min(sq.s_k, p.causal ? i + diag + 1 : sq.s_k);   // keys < lim_row allowed
      float m_true = -INFINITY;                   // running max (log2 units): the skip test
      float m_used = -INFINITY;                   // reference max of the exponentials
      float l = 0.f;
      bool pv_any = false;

      // One K/V tile: the four 32-key sub-tile maxima, the running max and
      // lazy rescale, then the exponentials in two halves; P of keys [0, 64)
      // is handed to the MMA warp before the second half is computed, so the
      // first half of P.V overlaps it.  (Starting the first half's
      // exponentials before the maxima, with a redo when a row's max grew,
      // measured 6 % slower: the maxima then trailed the exponentials on the
      // path to the hand-off.)  Skip mode: each warp votes per 32-key
      // sub-tile from its rows' maxima; the four votes are combined before
      // the exponentials, and a skipped sub-tile gets none: its p are 0, it
      // adds nothing to the row sums, and the MMA warp issues no P.V for it.
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      if (SKIP && quad == 0 && g.n > 0) n_vis += (g.k_end + kSkipTile - 1) / kSkipTile;
      auto step = [&](int j) -> bool {
        const bool ok =
            __all_sync(0xffffffffu, alive && wait_or_abort(&s_full[t], tile_c & 1, abort_flag, p.err));
        if (!ok) {
          alive = false;
          return false;
        }
        uint32_t sr[4][32];
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) tie(sr[c]);
        const int kbase = j * BN;
        if (kbase + BN > g.full_vis) mask_cols(sr, lim_row - kbase);
        float mref = (m_used == -INFINITY) ? 0.f : m_used;
        float um[4];                                // raw maxima of the four 32-key sub-tiles
        max_sub4(sr, um);
        uint32_t wv = 0;                            // sub-tiles every row of this warp votes to skip
        if constexpr (SKIP) {
          // vote per 32-key sub-tile: exp(sub-tile max - running max) <
          // threshold for every row of the warp
          uint32_t my_votes = 0;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float t2 = um[u] * sl2;
            const bool vote = !row_valid || (t2 == -INFINITY) || (t2 - m_true < p.thr_log2);
            m_true = fmaxf(m_true, t2);
            my_votes |= uint32_t(vote) << u;
          }
          wv = __reduce_and_sync(0xffffffffu, my_votes);
          if (lane == 0) {
            votes[(t * 3 + tile_c % 3) * 4 + quad] = wv;
            mbar_arrive(&votes_ready[2 * t + (tile_c & 1)]);
          }
        } else {
          m_true = fmaxf(m_true, fmaxf(fmaxf(um[0], um[1]), fmaxf(um[2], um[3])) * sl2);
        }
        // lazy rescale: move the reference max only when it grew by more than 2^8
        float alpha = 1.f;
        const bool grow = m_true > m_used + kRescaleLog2 || (m_used == -INFINITY && m_true > -INFINITY);
        if (grow) {
          alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_true);
          m_used = m_true;
          mref = m_used;
        }
        uint32_t skip = 0;                          // sub-tiles every row of the warpgroup skips
        if constexpr (SKIP) {
          // the four warps' votes (a warp is at most one tile ahead of the
          // others: the next S needs every warp's P of this one).  A sub-tile
          // is skipped only if every warp's word has its bit: a warp whose own
          // word is 0 knows that none is and does not wait for the others.
          if (wv != 0) {
            if (!__all_sync(0xffffffffu, wait_or_abort(&votes_ready[2 * t + (tile_c & 1)], (tile_c >> 1) & 1,
                                                       abort_flag, p.err))) {
              alive = false;
              return false;
            }
            skip = and4_shared(votes + (t * 3 + tile_c % 3) * 4);
          }
#pragma unroll
          for (int u = 0; u < 2; ++u)
            ps[u] = ((skip >> u) & 1u) ? 0.f : exp32_to_tmem(sr[u], sl2, mref, tS + 16 * u);
        } else {
          exp64_to_tmem(sr[0], sr[1], sl2, mref, tS, ps);
        }
        // rescale the O accumulator rows whose reference max moved
        if (pv_any && __any_sync(0xffffffffu, alpha != 1.f)) {
          const bool okw =
              __all_sync(0xffffffffu, wait_or_abort(&o_done[t], (tile_c - 1) & 1, abort_flag, p.err));
          if (!okw) alive = false;
          if (okw) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
              tie(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + c * 32, o);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_half[t]);
        if constexpr (SKIP) {
#pragma unroll
          for (int u = 2; u < 4; ++u)
            ps[u] = ((skip >> u) & 1u) ? 0.f : exp32_to_tmem(sr[u], sl2, mref, tS + 16 * u);
        } else {
          exp64_to_tmem(sr[2], sr[3], sl2, mref, tS + 32, ps + 2);
        }
        l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t]);
        if constexpr (SKIP) {
          // count and record the skipped units (sub-tiles past the keys vote
          // skip too, but are not units)
          if (quad == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (j * BN + 32 * u >= g.k_end) skip &= ~(1u << u);
            n_skip += __popc(skip);
            if (lane == 0 && p.skip_mask && skip != 0) {
              for (int u = 0; u < 4; ++u) {
                if ((skip >> u) & 1u) {
                  const long long unit = (((long long)it.b * p.qb_max + it.r[t]) * p.h_q + hq) * p.kt_max +
                                         (j * BN / 32 + u);
                  atomicOr(p.skip_mask + (unit >> 5), 1u << (unit & 31));
                }
              }
            }
          }
        }
        ++tile_c;
        pv_any = true;
        return alive;
      };

      for (int j = 0; j < g.n; ++j)
        if (!step(j)) break;
      if (!alive) break;

      // ---------------- epilogue ----------------
      const bool have_o = g.n > 0;
      if (have_o) {
        alive = __all_sync(0xffffffffu, wait_or_abort(&o_done[t], (tile_c - 1) & 1, abort_flag, p.err));
        if (!alive) break;
        tc_fence_after();
      }
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      if (have_o && g.r0 + BM <= sq.s_q) {
        // A full 128-row tile: normalised rows go, 64 columns at a time, to this
        // warpgroup's staging buffer in the store box's 128-byte-swizzled
        // layout, and one thread writes each box with a TMA store, so the
        // warps move on to the next item instead of waiting on 256-byte
        // scattered row stores.
        uint8_t *stg = sm + L::kStage + t * L::kStageBytes;
        const bool issuer = quad == 0 && lane == 0;
#pragma unroll 1
        for (int hh = 0; hh < D / 64; ++hh) {
          uint32_t o[2][32];
          tmem_ld32(tO + hh * 64, o[0]);
          tmem_ld32(tO + hh * 64 + 32, o[1]);
          tmem_wait_ld();
          tie(o[0]);
          tie(o[1]);
          if (hh == D / 64 - 1) {
            // the accumulator is free for the next item once the last columns are read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_free[t]);
          }
          if (issuer) bulk_wait_read();              // the previous box has left the buffer
          named_bar_sync(1 + t, 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t *v = &o[c >> 2][(c & 3) * 8];
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv);
            *reinterpret_cast<uint4 *>(stg + sw128_offset((uint32_t)row, (uint32_t)c)) = w;
          }
          fence_proxy_async_smem();
          named_bar_sync(1 + t, 128);
          if (issuer) {
            tma_store_3d(&omap, stg, hh * 64, hq, sq.q0 + g.r0);
            bulk_commit();
          }
        }
      } else {
        uint16_t *orow = p.out + ((size_t)(sq.q0 + i) * p.h_q + hq) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (have_o) {
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
            tie(o);
            if (c == D / 32 - 1) {
              // the accumulator is free for the next item once the last chunk is read
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&o_free[t]);
            }
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
      }
      if (row_valid && p.lse)
        p.lse[(size_t)(sq.q0 + i) * p.h_q + hq] = (l > 0.f) ? (m_used + __log2f(l)) * kLn2 : -INFINITY;
    }
    if (quad == 0 && lane == 0) bulk_wait_all();   // output boxes written before the CTA ends
    if (SKIP && quad == 0 && lane == 0 && p.skip_counts) {
      atomicAdd(p.skip_counts + 0, n_vis);
      atomicAdd(p.skip_counts + 1, n_skip);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// SM count of the current device, looked up once per device.
int num_sms() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> count[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  if (dev >= kMaxDevices) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 1;
  }
  int n = count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 1;
    count[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int D, bool SKIP, bool PAGED>
cudaError_t launch_t(const PrefillParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                     const CUtensorMap &vmap, const CUtensorMap &omap, cudaStream_t stream) {
  const int smem = Smem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, SKIP, PAGED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long items = (p.group % 2 == 0) ? (long long)p.batch * p.qb_max * (p.h_q / 2)
                                             : (long long)p.batch * ((p.qb_max + 1) / 2) * p.h_q;
  const int grid = (int)(items < num_sms() ? items : num_sms());
  // a nonzero tag per launch; launches take the claim slots in turn
  static std::atomic<unsigned int> next_tag{0};
  PrefillParams q = p;
  q.work_tag = next_tag.fetch_add(1u) % 0xffffffffu + 1u;
  q.work_slot = (int)(q.work_tag % kWorkSlots);
  prefill_kernel<D, SKIP, PAGED><<<grid, kThreads, smem, stream>>>(qmap, kmap, vmap, omap, q);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &qmap, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, const CUtensorMap &omap, cudaStream_t stream) {
  if (p.batch == 0 || p.qb_max == 0) return cudaSuccess;
  const bool skip = p.thr_log2 > -INFINITY;
  // one instantiation per (head dim, skip, paged): each keeps only its own
  // load and softmax code
  auto go = [&](auto d, auto sk) {
    return p.paged ? launch_t<decltype(d)::value, decltype(sk)::value, true>(p, qmap, kmap, vmap, omap, stream)
                   : launch_t<decltype(d)::value, decltype(sk)::value, false>(p, qmap, kmap, vmap, omap, stream);
  };
  using T = std::true_type;
  using F = std::false_type;
  if (p.d == 128)
    return skip ? go(std::integral_constant<int, 128>{}, T{}) : go(std::integral_constant<int, 128>{}, F{});
  return skip ? go(std::integral_constant<int, 64>{}, T{}) : go(std::integral_constant<int, 64>{}, F{});
}

}  // namespace attn
