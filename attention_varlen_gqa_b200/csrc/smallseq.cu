// smallseq.cu -- s_q = 1, s_kv <= 16 cross attention (sm_100a).
//
// ROCm/TransformerEngine PR 461 ("Integrate CK varlen cross attention for
// small-seq (s_q=1, s_kv<=16)") runs this case as three kernels (scores,
// mask + softmax, output) with runtime dispatch over max_seqlen_kv in
// {2,4,6,8,12,16}; the batch counts query tokens.  Here it is one fused,
// memory-bound kernel: every byte of Q, K and V is read once.
//
// A unit is (query token t, group of up to 16 heads).  Its bytes are the
// group's query rows and, for each of the token's keys, the group's K and V
// rows; with the heads in one group (h <= 16) a token's K (and V) rows of
// all keys are one contiguous run of the packed [keys, heads, d] tensor.  One
// persistent CTA per SM streams its units through a shared-memory byte ring:
// a producer warp issues bulk asynchronous copies (one each for Q, K and V
// of a token, or one per key when the heads span several groups) completing
// on the unit's mbarrier, so the copies of the next units are in flight while
// the current one is computed and no load waits in a register.  Sixteen
// consumer warps take one head of the unit each: lane i holds dims [d/32 i,
// d/32 (i + 1)) read from shared memory, the <= 16 partial dot products are
// reduced across the warp by a reduce-scatter shuffle tree (16 shuffles for
// 16 keys instead of 80), and softmax, weights and O = P V stay in registers.
// The row's own key count picks the code path (up to 4, 8 or 16 keys).
// Tokens are split between CTAs in equal shares of their bytes (2 + 2 s_kv
// head rows a token) by a search over cu_seqlens_kv, so every CTA streams one
// contiguous range of memory.
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kHeads = 16;                       // heads per unit = consumer warps
constexpr int kThreads = 32 * (kHeads + 1);      // + the producer warp
constexpr int kDesc = 16;                        // units in flight (descriptor slots)
constexpr uint32_t kRing = 224 * 1024;           // bytes of the unit ring
constexpr int kProbe = 256;                      // probes per round of the partition search

// n >= 0: key count; kBadRange / kTooLong: the row is written as zeros.
// k0: the token's first key; off: the unit's byte offset in the ring.
struct Unit {
  int token, group, n, off, k0;
};
constexpr int kBadRange = -1;
constexpr int kTooLong = -2;

struct Layout {
  static constexpr uint32_t kDescOff = kRing;                        // [kDesc] Unit
  static constexpr uint32_t kFull = kDescOff + kDesc * sizeof(Unit); // [kDesc] the unit's bytes landed
  static constexpr uint32_t kEmpty = kFull + kDesc * 8;              // [kDesc] its consumers are done
  static constexpr uint32_t kStart = kEmpty + kDesc * 8;             // [kDesc] ring position (producer)
  static constexpr uint32_t kScratch = kStart + kDesc * 8;           // partition search
  static constexpr size_t kBytes = kScratch + 16 + 128;              // + alignment slack
};
static_assert(Layout::kBytes <= 227 * 1024, "fits one CTA per SM");

template <int D>
struct LaneVec;
template <>
struct LaneVec<128> {   // 4 bf16 per lane
  using T = uint2;
  static constexpr int E = 4;
  static ATTN_DEVICE T lds(uint32_t a) {
    T r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
    return r;
  }
  static ATTN_DEVICE void unpack(const T &x, float *f) {
    f[0] = bf16_lo(x.x); f[1] = bf16_hi(x.x); f[2] = bf16_lo(x.y); f[3] = bf16_hi(x.y);
  }
  static ATTN_DEVICE T pack(const float *f) { return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3])); }
};
template <>
struct LaneVec<64> {    // 2 bf16 per lane
  using T = uint32_t;
  static constexpr int E = 2;
  static ATTN_DEVICE T lds(uint32_t a) {
    T r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(a));
    return r;
  }
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

// One (query token, head) row with 0 < n <= NK keys, read from its unit in
// shared memory: q at qa, key j's K row at ka + j * kstride, V row at
// va + j * kstride (addresses already offset by this lane's dims).
template <int D, int NK>
ATTN_DEVICE void row_attention(const SmallSeqParams &p, uint32_t qa, uint32_t ka, uint32_t va,
                               uint32_t kstride, int n, size_t row, int lane) {
  using LV = LaneVec<D>;
  using T = typename LV::T;
  constexpr int E = LV::E;
  static_assert(NK == 4 || NK == 8 || NK == 16, "power-of-two key counts for the reduce-scatter");
  constexpr int SH = (NK == 16) ? 1 : (NK == 8) ? 2 : 3;  // key of lane l after the reduce-scatter is l >> SH
  T kr[NK], vr[NK];
  const T qv = LV::lds(qa);
#pragma unroll
  for (int j = 0; j < NK; ++j)
    if (j < n) kr[j] = LV::lds(ka + j * kstride);
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
  float m = (key < n) ? sc * p.scale_log2 : -INFINITY;
  const float s2 = m;
  // every key sits in 2^SH neighbouring lanes: the lane bits from SH up span each key once
#pragma unroll
  for (int o = 16; o >= (1 << SH); o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float pr = (key < n) ? ex2(s2 - m) : 0.f;
  float l = pr;
#pragma unroll
  for (int o = 16; o >= (1 << SH); o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  const float inv = 1.f / l;
#pragma unroll
  for (int j = 0; j < NK; ++j)
    if (j < n) vr[j] = LV::lds(va + j * kstride);
  float o_acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o_acc[e] = 0.f;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const float pj = __shfl_sync(0xffffffffu, pr, j << SH);
    if (j < n) {
      float vf[E];
      LV::unpack(vr[j], vf);
#pragma unroll
      for (int e = 0; e < E; ++e) o_acc[e] = fmaf(pj, vf[e], o_acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) o_acc[e] *= inv;
  reinterpret_cast<T *>(p.out + row * D)[lane] = LV::pack(o_acc);
  if (p.weights) {
    const float pt = __shfl_sync(0xffffffffu, pr, (lane < NK ? lane : 0) << SH);
    if (lane < p.max_s_kv) p.weights[row * p.max_s_kv + lane] = f32_to_bf16(lane < n ? pt * inv : 0.f);
  }
}

// Backward of one (query token, head) row with 0 < n <= NK keys, from its
// unit in shared memory (q at qa, dO at oa, key j's K and V rows at ka, va +
// j * kstride) and the forward's weights (lane j < NK holds P_j).  The steps
// of ROCm/TransformerEngine PR 461's backward:
//   grad_attn     dP_j = <dO, v_j>            (reduce-scattered: lane l, key l >> SH)
//   softmax bwd   dS_j = P_j (dP_j - sum_i P_i dP_i)
//   grad_V        dV_j = P_j dO               (row j of dv)
//   grad_K        dK_j = scale dS_j q         (row j of dk)
//   grad_Q        dQ   = scale sum_j dS_j k_j
// Key j's rows of this head start at element kv0 + j * kvs of dk and dv.
template <int D, int NK>
ATTN_DEVICE void row_backward(const SmallSeqParams &p, uint32_t qa, uint32_t oa, uint32_t ka, uint32_t va,
                              uint32_t kstride, int n, float pw, size_t row, size_t kv0, size_t kvs,
                              int lane) {
  using LV = LaneVec<D>;
  using T = typename LV::T;
  constexpr int E = LV::E;
  static_assert(NK == 4 || NK == 8 || NK == 16, "power-of-two key counts for the reduce-scatter");
  constexpr int SH = (NK == 16) ? 1 : (NK == 8) ? 2 : 3;
  float q[E], dO[E];
  LV::unpack(LV::lds(qa), q);
  LV::unpack(LV::lds(oa), dO);
  T r[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j)
    if (j < n) r[j] = LV::lds(va + j * kstride);
  float part[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    float vf[E];
    LV::unpack(r[j], vf);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc = fmaf(dO[e], vf[e], acc);
    part[j] = (j < n) ? acc : 0.f;
  }
  const int key = lane >> SH;
  const float dp = reduce_scatter<NK>(part, lane);
  const float pk = __shfl_sync(0xffffffffu, pw, key);
  float t = (key < n) ? pk * dp : 0.f;
#pragma unroll
  for (int o = 16; o >= (1 << SH); o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  const float ds = (key < n) ? pk * (dp - t) : 0.f;
#pragma unroll
  for (int j = 0; j < NK; ++j)
    if (j < n) r[j] = LV::lds(ka + j * kstride);
  float dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) dq[e] = 0.f;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const float pj = __shfl_sync(0xffffffffu, pw, j);
    const float dsj = __shfl_sync(0xffffffffu, ds, j << SH);
    if (j < n) {
      float a[E], kf[E];
      const size_t at = kv0 + j * kvs;
#pragma unroll
      for (int e = 0; e < E; ++e) a[e] = pj * dO[e];
      reinterpret_cast<T *>(p.dv + at)[lane] = LV::pack(a);
      const float sk = p.scale * dsj;
#pragma unroll
      for (int e = 0; e < E; ++e) a[e] = sk * q[e];
      reinterpret_cast<T *>(p.dk + at)[lane] = LV::pack(a);
      LV::unpack(r[j], kf);
#pragma unroll
      for (int e = 0; e < E; ++e) dq[e] = fmaf(dsj, kf[e], dq[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) dq[e] *= p.scale;
  reinterpret_cast<T *>(p.dq + row * D)[lane] = LV::pack(dq);
}

// Token boundary of CTA c of G: the first t in [0, T] with g(t) >= X_c, where
// g(t) = wt t + wk cu[t] counts the head rows moved before token t (wt a
// token, wk a key: 2 and 2 forward, 3 and 4 backward) and X_c = c / G of
// g(T); boundary 0 is 0 and boundary G is T.
// Threads [0, kProbe) search this CTA's first boundary and [kProbe,
// 2 kProbe) its last, each round probing kProbe evenly spaced tokens of the
// current bracket.  For valid (non-decreasing) cu the result is exact; for
// any cu, consecutive CTAs' ranges still cover [0, T), since boundary 0 is 0
// and boundary G is T.
ATTN_DEVICE void token_range(const SmallSeqParams &p, int wt, int wk, int *scratch, int &t0, int &t1) {
  const int tid = threadIdx.x;
  const int T = p.batch;
  const int G = gridDim.x;
  const int side = tid / kProbe;
  const int pi = tid % kProbe;
  const bool searcher = side < 2;
  const int c = blockIdx.x + side;
  int lo = 0, hi = T;            // the boundary lies in [lo, hi]; hi satisfies (or is T)
  long long X = 0;
  bool done = !searcher;
  if (searcher) {
    if (c == 0) {
      hi = 0;
      done = true;
    } else if (c >= G) {
      lo = T;
      done = true;
    } else {
      const long long total = (long long)wt * T + (long long)wk * __ldg(p.cu + T);
      X = total * c / G;
    }
  }
  while (__syncthreads_or(!done)) {
    if (tid < 2) scratch[tid] = INT_MAX;
    __syncthreads();
    const int span = hi - lo;
    const int step = done ? 1 : (span + kProbe - 1) / kProbe;
    const long long cand = lo + (long long)pi * step;
    if (!done && cand < hi) {
      const int t = (int)cand;
      if ((long long)wt * t + (long long)wk * __ldg(p.cu + t) >= X) atomicMin(&scratch[side], pi);
    }
    __syncthreads();
    if (!done) {
      const int f = scratch[side];
      if (f == INT_MAX) {
        lo += ((span + step - 1) / step - 1) * step + 1;   // past the last probe
      } else {
        hi = lo + f * step;
        lo = (f == 0) ? hi : lo + (f - 1) * step + 1;
      }
      done = lo >= hi;
    }
  }
  if (pi == 0 && searcher) scratch[2 + side] = lo;
  __syncthreads();
  t0 = scratch[2];
  t1 = scratch[3];
}

// BWD: the backward (units carry q, dO, K, V; consumers run row_backward).
template <int D, bool BWD>
__global__ void __launch_bounds__(kThreads, 1) smallseq_kernel(SmallSeqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  Unit *desc = reinterpret_cast<Unit *>(base + Layout::kDescOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(base + Layout::kFull);
  uint64_t *empty = reinterpret_cast<uint64_t *>(base + Layout::kEmpty);
  uint64_t *ustart = reinterpret_cast<uint64_t *>(base + Layout::kStart);
  int *scratch = reinterpret_cast<int *>(base + Layout::kScratch);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.h;
  const int ngroups = (H + kHeads - 1) / kHeads;
  constexpr uint32_t kRow = D * 2;   // bytes of one head row
  constexpr uint32_t kQRows = BWD ? 2 : 1;   // query-side rows of a unit: q (and dO)

  if (tid == 0) {
    for (int s = 0; s < kDesc; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kHeads);
    }
    fence_barrier_init();
  }
  int t0, t1;
  token_range(p, BWD ? 3 : 2, BWD ? 4 : 2, scratch, t0, t1);   // its barriers also publish the mbarrier init
  const long long units = (long long)max(0, t1 - t0) * ngroups;

  if (warp == kHeads) {
    // ------------------------------ producer ------------------------------
    // lane l holds cu[wb + l] and cu[wb + 32 + l]; lane 0 issues and keeps the ring
    auto ld_cu = [&](int i) { return i <= p.batch ? __ldg(p.cu + i) : 0; };
    int wb = t0;
    int c_cur = ld_cu(wb + lane), c_nxt = ld_cu(wb + 32 + lane);
    uint64_t hb = 0;            // ring bytes handed out so far
    long long i = 0, o = 0;     // units issued / units known released
    bool ok = true;
    for (int t = t0; t < t1 && ok; ++t) {
      if (t - wb == 32) {
        wb += 32;
        c_cur = c_nxt;
        c_nxt = ld_cu(wb + 32 + lane);
      }
      const int j = t - wb;
      const int k0 = __shfl_sync(0xffffffffu, c_cur, j);
      const int k1 = __shfl_sync(0xffffffffu, j < 31 ? c_cur : c_nxt, (j + 1) & 31);
      const int n = k1 - k0;
      const bool bad = (k0 < 0) | (n < 0) | (k1 > p.total_kv);
      const bool too_long = !bad && n > p.max_s_kv;
      const int ncode = bad ? kBadRange : (too_long ? kTooLong : n);
      if (lane == 0) {
        if (bad) raise_error(p.err, ATTN_DEVERR_CU_SEQLENS);
        if (too_long) raise_error(p.err, ATTN_DEVERR_SMALLSEQ_LEN);
      }
      for (int g = 0; g < ngroups && ok; ++g) {
        const int hg = min(kHeads, H - g * kHeads);
        const uint32_t row = hg * kRow;
        const uint32_t bytes = ncode > 0 ? row * (kQRows + 2 * n) : 0u;
        uint64_t start = hb;
        if (bytes != 0 && (hb % kRing) + bytes > kRing) start = hb + (kRing - hb % kRing);   // wrap
        if (lane == 0) {
          // release the oldest units until this one has a descriptor slot and room
          while (o < i && (i - o >= kDesc || start + bytes - ustart[o % kDesc] > kRing)) {
            if (!mbar_wait(&empty[o % kDesc], (uint32_t)(o / kDesc) & 1u, p.err)) {
              ok = false;
              break;
            }
            ++o;
          }
          if (ok) {
            const int s = (int)(i % kDesc);
            const uint32_t off = (uint32_t)(start % kRing);
            desc[s] = Unit{t, g, ncode, (int)off, k0};
            ustart[s] = start;
            mbar_arrive_expect_tx(&full[s], bytes);
            if (bytes != 0) {
              uint8_t *dst = base + off;
              const size_t qsrc = ((size_t)t * H + g * kHeads) * D;
              bulk_load(dst, p.q + qsrc, row, &full[s]);
              if (BWD) bulk_load(dst + row, p.dout + qsrc, row, &full[s]);
              uint8_t *kd = dst + row * kQRows, *vd = kd + row * n;
              if (hg == H) {   // all heads in one group: the token's K (V) rows are one run
                bulk_load(kd, p.k + (size_t)k0 * H * D, row * n, &full[s]);
                bulk_load(vd, p.v + (size_t)k0 * H * D, row * n, &full[s]);
              } else {
                for (int jj = 0; jj < n; ++jj) {
                  const size_t src = ((size_t)(k0 + jj) * H + g * kHeads) * D;
                  bulk_load(kd + row * jj, p.k + src, row, &full[s]);
                  bulk_load(vd + row * jj, p.v + src, row, &full[s]);
                }
              }
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        hb = start + bytes;
        ++i;
      }
    }
    if (!ok && lane == 0) {
      // let the copies still in flight land before the shared memory goes away
      for (long long x = o; x < i; ++x) mbar_wait(&full[x % kDesc], (uint32_t)(x / kDesc) & 1u, nullptr);
    }
  } else {
    // ------------------------------ consumers ------------------------------
    const int w = warp;   // head of the unit's group
    const uint32_t sbase = smem_u32(base);
    using LV = LaneVec<D>;
    // backward: lane j < max_s_kv holds P_j of this warp's head of unit i + 1,
    // loaded one unit ahead (unit i is token t0 + i / ngroups, group i % ngroups)
    auto load_weights = [&](long long i) -> float {
      if (!BWD || i >= units || lane >= p.max_s_kv) return 0.f;
      const long long t = t0 + i / ngroups;
      const int hh = (int)(i % ngroups) * kHeads + w;
      if (hh >= H) return 0.f;
      return bf16_to_f32(__ldg(p.weights_in + ((size_t)t * H + hh) * p.max_s_kv + lane));
    };
    float pw_next = load_weights(0);
    for (long long i = 0; i < units; ++i) {
      const float pw = pw_next;
      pw_next = load_weights(i + 1);
      const int s = (int)(i % kDesc);
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(i / kDesc) & 1u, p.err))) break;
      const Unit u = desc[s];
      const int hg = min(kHeads, H - u.group * kHeads);
      if (w < hg) {
        const int hh = u.group * kHeads + w;
        const size_t row = (size_t)u.token * H + hh;
        const int n = u.n;
        float z[LV::E] = {};
        if (n <= 0) {
          if (BWD) {
            reinterpret_cast<typename LV::T *>(p.dq + row * D)[lane] = LV::pack(z);
          } else {
            reinterpret_cast<typename LV::T *>(p.out + row * D)[lane] = LV::pack(z);
            if (p.weights && lane < p.max_s_kv) p.weights[row * p.max_s_kv + lane] = 0;
          }
        } else {
          const uint32_t lo = lane * sizeof(typename LV::T);
          const uint32_t qa = sbase + u.off + w * kRow + lo;
          const uint32_t ka = sbase + u.off + kQRows * hg * kRow + w * kRow + lo;
          const uint32_t va = ka + n * hg * kRow;
          const uint32_t ks = hg * kRow;
          if (BWD) {
            const uint32_t oa = qa + hg * kRow;
            const size_t kv0 = ((size_t)u.k0 * H + hh) * D, kvs = (size_t)H * D;
            if (n <= 4)
              row_backward<D, 4>(p, qa, oa, ka, va, ks, n, pw, row, kv0, kvs, lane);
            else if (n <= 8)
              row_backward<D, 8>(p, qa, oa, ka, va, ks, n, pw, row, kv0, kvs, lane);
            else
              row_backward<D, 16>(p, qa, oa, ka, va, ks, n, pw, row, kv0, kvs, lane);
          } else {
            if (n <= 4)
              row_attention<D, 4>(p, qa, ka, va, ks, n, row, lane);
            else if (n <= 8)
              row_attention<D, 8>(p, qa, ka, va, ks, n, row, lane);
            else
              row_attention<D, 16>(p, qa, ka, va, ks, n, row, lane);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
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

template <int D, bool BWD>
cudaError_t launch_d(const SmallSeqParams &p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(smallseq_kernel<D, BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)Layout::kBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.batch < num_sms() ? p.batch : num_sms();   // at least one token a CTA
  smallseq_kernel<D, BWD><<<grid, kThreads, Layout::kBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_smallseq(const SmallSeqParams &p, cudaStream_t stream) {
  if ((long long)p.batch * p.h == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128, false>(p, stream) : launch_d<64, false>(p, stream);
}

cudaError_t launch_smallseq_bwd(const SmallSeqParams &p, cudaStream_t stream) {
  if ((long long)p.batch * p.h == 0) return cudaSuccess;
  return p.d == 128 ? launch_d<128, true>(p, stream) : launch_d<64, true>(p, stream);
}

}  // namespace attn
