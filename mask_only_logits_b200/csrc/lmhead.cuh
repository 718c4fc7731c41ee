// lmhead.cuh - masked_lmhead: the mask-only LM head on the 5th-generation tensor cores with
// the softmax statistics fused into the epilogue (Mosaic page, TL;DR and Abstract: the
// mask-only logits kernel; the logits of the masked rows are never written either).
//
// C[i, v] = sum_k Hm[i, k] * W[v, k] for the compacted masked rows Hm (bf16, K-major) and
// the vocabulary projection W (bf16, K-major), fp32 accumulation in tensor memory.
//
// Persistent, warp-specialised GEMM, one CTA per SM, 192 threads, in two bodies (the
// device function lmhead_run, templated on the CTA group size CG):
//   CG = 1  each CTA owns a 128 x 256 tile (tcgen05.mma.cta_group::1, M=128, N=256)
//   CG = 2  a cluster of two CTAs on paired SMs owns a 256 x 256 tile
//           (tcgen05.mma.cta_group::2, M=256, N=256): each CTA stages 128 rows of Hm and
//           128 rows of W per stage, the leader CTA issues the MMAs for both, and each CTA's
//           TMEM holds its own 128 rows of the accumulator.  Per SM this halves the W bytes
//           staged per flop.
// lmhead_auto_kernel (the default) is launched in clusters of two CTAs and picks the body
// on the device from the masked count; lmhead_kernel<CG> runs one body fixed at launch.
// Roles (per CTA):
//   warp 0      TMA producer: a 128x64 tile of Hm and a (256/CG)x64 tile of W per stage
//               (128-byte swizzle) into a kStages-deep shared-memory ring
//   warp 1      allocates 512 TMEM columns; lane 0 of the leader issues the MMAs (four per
//               stage) into one of two 256-column fp32 accumulators and commits stage
//               releases / accumulator-full events to mbarriers
//   warps 2..5  epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (one row per thread) with
//               tcgen05.ld, keeps a running (max, sum exp(z - max), first argmax) per row
//               over the vocabulary tiles of its unit, then writes one partial per row
//
// Work decomposition.  A "unit" is (m-tile, contiguous range of vocabulary tiles).  m-tiles
// are taken in groups of up to `gmax`; inside a group of G m-tiles the work holders (CTAs,
// or CTA pairs for CG = 2) are split into P = floor(holders / G) vocabulary streams, holder
// c handling m-tile c % G and stream c / G.  Holders of one stream therefore walk the same
// W tiles at the same time (each W tile is fetched from HBM about once per group and served
// from L2 to the others) while the group's Hm tiles stay resident in L2.  Per row, the
// partials of the P streams are merged (lse_merge) by the epilogue of whichever CTA finishes
// the m-tile's last unit (its four epilogue warps each merge a quarter of the partials, then
// combine in order); with P = 1 the unit's statistics are the result.  A problem of one
// m-tile takes the fewest streams that keep the busiest stream's tile count; the other
// holders stay idle (B1 L4096 with 64 masked rows: 0.190 against 0.199 ms per step).
//
// Every wait is bounded (ptx.cuh).  On a timeout the CTA raises its abort flag, every role
// unwinds, the MMA issuer waits (bounded) for its issued MMAs, the producer of the CTA that
// arms the stages waits (bounded) for the full barrier of the last phase it armed on every
// stage, so that no TMA load is still writing shared memory, and TMEM is released before
// the kernel returns.
#pragma once
#include "ptx.cuh"

// Compile-time tuning knobs (defaults are the measured best).
#ifndef DLLM_GROUP_M1
#define DLLM_GROUP_M1 37          // m-tiles per L2 group, single-CTA variant
#endif
#ifndef DLLM_GROUP_M2
#define DLLM_GROUP_M2 18          // m-tiles per L2 group, CTA-pair variant
#endif
#ifndef DLLM_STAGES2
#define DLLM_STAGES2 6            // shared-memory ring depth, CTA-pair variant
#endif
#ifndef DLLM_REMAINDER_HOLDERS
#define DLLM_REMAINDER_HOLDERS 1  // give the last vocabulary columns to otherwise idle holders
#endif
#ifndef DLLM_EPI_BACKOFF_NS
#define DLLM_EPI_BACKOFF_NS 0     // epilogue: sleep between polls of the accumulator barrier
#endif
#ifndef DLLM_FEWEST_STREAMS
#define DLLM_FEWEST_STREAMS 1     // one m-tile: fewest streams with the same busiest tile count
#endif
#ifndef DLLM_PAIR_PACE
#define DLLM_PAIR_PACE 2          // CTA-pair body: lead a holder may take over its stream, in
#endif                            // tiles (0 = no pacing)

namespace dllm {
namespace lm {

constexpr int BN = 256;                 // vocabulary entries per tile (UMMA N)
constexpr int BK = 64;                  // K per stage: one 128-byte swizzle atom of bf16
constexpr int UK = 16;                  // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 2 * BN;       // two accumulators
constexpr int kMaxCtas = 160;           // partial-buffer sizing bound (B200: 148 SMs)
constexpr float kLog2e = 1.4426950408889634f;

template <int CG>
struct Cfg {
  static_assert(CG == 1 || CG == 2, "CTA group of 1 or 2");
  static constexpr int BM_CTA = 128;                 // rows per CTA (TMEM lanes)
  static constexpr int BM = BM_CTA * CG;             // rows per m-tile
  static constexpr int B_ROWS = BN / CG;             // W rows staged per CTA per stage
  static constexpr int A_BYTES = BM_CTA * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int kStages = CG == 1 ? 4 : DLLM_STAGES2;
  // ring, barriers and flags, and the merge's combine buffer (4 x 128 row states)
  static constexpr int kCombBytes = 4 * BM_CTA * 20;
  static constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + 256 + kCombBytes;
  static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory of one CTA");
  static constexpr int kGroupM = CG == 1 ? DLLM_GROUP_M1 : DLLM_GROUP_M2;  // m-tiles per L2 group
  // Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B bf16
  // (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22,
  // M >> 4 at bits 24-28.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (static_cast<uint32_t>(BN >> 3) << 17) |
                                     (static_cast<uint32_t>(BM >> 4) << 24);
};

// The unit schedule, computed identically by every role of the GEMM (and by host code).
//
// m-tiles are taken in groups of up to gmax.  Inside a group of G m-tiles each holder takes
// one m-tile and a contiguous range of vocabulary tiles: P = ctas / G "streams" per m-tile,
// holder h on m-tile h % G and stream h / G, so the holders of one stream walk the same W
// tiles at the same time and each W tile is fetched from HBM about once per group.
//
// Remainder holders (a problem that fits one group, when G does not divide the holders):
// the streams take exactly rb = numN / P tiles each, and the last rr = numN - P * rb
// vocabulary columns of every m-tile (G * rr tiles, in m-major order) are split among the
// R = ctas - G * P holders the streams leave idle.  Every holder then runs at most
// max(rb, ceil(G * rr / R)) tiles instead of ceil(numN / P).
struct Plan {
  int count, bm, numM, numN, ctas, gmax, ngroups, P_full;
  bool rem;        // remainder holders in use (implies ngroups == 1)
  int R, rb, rr;

  // ctas = number of work holders (CTAs for CG = 1, CTA pairs for CG = 2);
  // bm = rows per m-tile.
  __host__ __device__ static Plan make(int count, int V, int ctas, int gmax, int bm) {
    Plan p;
    p.count = count;
    p.bm = bm;
    p.numM = (count + bm - 1) / bm;
    p.numN = (V + BN - 1) / BN;
    p.ctas = ctas;
    p.gmax = gmax < ctas ? gmax : ctas;
    p.ngroups = (p.numM + p.gmax - 1) / p.gmax;
    p.P_full = streams(p.gmax, p.ctas, p.numN);
    p.rem = false;
    p.R = p.rb = p.rr = 0;
    if (DLLM_REMAINDER_HOLDERS && p.ngroups == 1) {
      const int G = p.numM, P = streams(G, ctas, p.numN);
      const int R = ctas - G * P, rb = p.numN / P, rr = p.numN - P * rb;
      // only when it shortens the busiest holder: max(rb, ceil(G rr / R)) < ceil(numN / P)
      const int busiest_rem = R > 0 ? (rb > (G * rr + R - 1) / R ? rb : (G * rr + R - 1) / R) : 0;
      if (R > 0 && rr > 0 && busiest_rem < rb + 1) {
        p.rem = true;
        p.R = R;
        p.rb = rb;
        p.rr = rr;
      }
    }
    return p;
  }
  __host__ __device__ static int streams(int G, int ctas, int numN) {
    int P = ctas / G;
    if (P > numN) P = numN;
    if (P < 1) P = 1;
#if DLLM_FEWEST_STREAMS
    // one m-tile: the fewest streams that keep the busiest one's tile count (594 tiles on 74
    // CTA pairs: 66 streams of exactly 9 instead of 72 of 8 and 2 of 9); the holders left
    // over stay idle and leave the power to the others
    if (G == 1) {
      const int per = (numN + P - 1) / P;
      P = (numN + per - 1) / per;
    }
#endif
    return P;
  }
  __host__ __device__ int group_size(int g) const {
    return g == ngroups - 1 ? numM - g * gmax : gmax;
  }
  // Partial-buffer index of (group g of size G, slot, row r within the group).  Slots:
  // streams 0..P-1, then remainder holders P..P+R-1.
  __host__ __device__ long long part_index(int g, int G, int slot, int r) const {
    return static_cast<long long>(g) * gmax * bm * P_full + static_cast<long long>(slot) * G * bm + r;
  }
  // Number of partial entries written for this count.
  __host__ __device__ long long part_entries() const {
    if (ngroups == 0) return 0;
    const int Gl = group_size(ngroups - 1);
    const int slots = streams(Gl, ctas, numN) + (rem ? R : 0);
    return part_index(ngroups - 1, Gl, 0, 0) + static_cast<long long>(Gl) * bm * slots;
  }
  // Remainder holder j: its tiles [i0, i1) of the m-major remainder list, tile i being
  // vocabulary column P * rb + i % rr of m-tile i / rr.
  __host__ __device__ void leftover_range(int j, int G, long long& i0, long long& i1) const {
    const long long T = static_cast<long long>(G) * rr;
    i0 = T * j / R;
    i1 = T * (j + 1) / R;
  }
  // Remainder holders whose tiles include m-tile m: j_lo..j_hi (none if j_lo > j_hi).
  __host__ __device__ void leftovers_of(int m, int G, int& j_lo, int& j_hi) const {
    j_lo = R;
    j_hi = -1;
    for (int j = 0; j < R; ++j) {
      long long i0, i1;
      leftover_range(j, G, i0, i1);
      if (i1 > i0 && i0 < static_cast<long long>(m + 1) * rr && i1 > static_cast<long long>(m) * rr) {
        if (j < j_lo) j_lo = j;
        j_hi = j;
      }
    }
  }
};

// The unit of a holder inside group g: a stream (one m-tile, vocabulary tiles [n0, n1)) or a
// remainder holder (remainder tiles [i0, i1)); false if the holder is idle in this group.
struct Unit {
  int m_tile, m_local, G, p, P, n0, n1;
  bool leftover;
  long long i0, i1;
};
__host__ __device__ __forceinline__ bool unit_of(const Plan& pl, int g, int holder, Unit& u) {
  u.G = pl.group_size(g);
  u.P = Plan::streams(u.G, pl.ctas, pl.numN);
  u.leftover = false;
  if (holder < u.G * u.P) {
    u.m_local = holder % u.G;
    u.m_tile = g * pl.gmax + u.m_local;
    u.p = holder / u.G;
    if (pl.rem) {
      u.n0 = u.p * pl.rb;
      u.n1 = u.n0 + pl.rb;
    } else {
      u.n0 = static_cast<int>(static_cast<long long>(u.p) * pl.numN / u.P);
      u.n1 = static_cast<int>(static_cast<long long>(u.p + 1) * pl.numN / u.P);
    }
    return true;
  }
  if (pl.rem && holder < u.G * u.P + pl.R) {
    const int j = holder - u.G * u.P;
    u.leftover = true;
    u.p = u.P + j;
    pl.leftover_range(j, u.G, u.i0, u.i1);
    return u.i1 > u.i0;
  }
  return false;
}

// Calls f(m_tile, n) for every tile of the holder, in order; stops early when f returns
// false.  Returns whether all calls returned true.
template <class F>
__host__ __device__ __forceinline__ bool for_each_tile(const Plan& pl, int holder, F& f) {
  for (int g = 0; g < pl.ngroups; ++g) {
    Unit u;
    if (!unit_of(pl, g, holder, u)) continue;
    if (u.leftover) {
      for (long long i = u.i0; i < u.i1; ++i)
        if (!f(g * pl.gmax + static_cast<int>(i / pl.rr), u.P * pl.rb + static_cast<int>(i % pl.rr)))
          return false;
    } else {
      for (int n = u.n0; n < u.n1; ++n)
        if (!f(u.m_tile, n)) return false;
    }
  }
  return true;
}

template <int CG>
struct Smem {
  uint8_t* a;          // kStages x A_BYTES
  uint8_t* b;          // kStages x B_BYTES
  uint64_t* full;      // kStages
  uint64_t* empty;     // kStages
  uint64_t* tfull;     // 2
  uint64_t* tempty;    // 2
  uint64_t* drain;     // 1: MMA completion on the abort path
  uint64_t* epi_bar;   // 1: barrier of the four epilogue warps (bounded, unlike bar.sync)
  uint32_t* tmem_slot;
  int* abort_flag;
  volatile int* last_flag;   // epilogue: this CTA finished the last unit of an m-tile
  struct RowStateRaw { float m, s, t, m2; int a; };
  RowStateRaw* comb;         // merge: per warp quarter, the merged state of each of 128 rows

  __device__ __forceinline__ explicit Smem(uint8_t* raw) {
    using C = Cfg<CG>;
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    a = base;
    b = base + C::kStages * C::A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(b + C::kStages * C::B_BYTES);
    full = bars;
    empty = bars + C::kStages;
    tfull = bars + 2 * C::kStages;
    tempty = bars + 2 * C::kStages + 2;
    drain = bars + 2 * C::kStages + 4;
    epi_bar = bars + 2 * C::kStages + 5;
    tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 6);
    abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
    last_flag = abort_flag + 1;
    comb = reinterpret_cast<RowStateRaw*>(reinterpret_cast<uint8_t*>(bars) + 256);
  }
};

// Epilogue modes: statistics for tok / lse / conf; the same plus the entropy and the
// top-2 probability margin of each row's softmax; or raw logits stored (test hook).
constexpr int kModeStats = 0;
constexpr int kModeStatsExt = 1;
constexpr int kModeDebugStore = 2;

// Running softmax statistics of one row over the vocabulary seen so far:
//   m  = max logit, a = its first index, s = sum exp(z - m),
//   t  = sum exp(z - m) (z - m)  (extended mode; entropy = ln s - t / s),
//   m2 = second-largest logit    (extended mode; margin p1 - p2 = (1 - exp(m2 - m)) / s).
struct RowState {
  float m, s, t, m2;
  int a;
  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    s = 0.f;
    t = 0.f;
    m2 = -INFINITY;
    a = 0;
  }
};

// Fold 32 consecutive logits (vocabulary columns col0..col0+31) into a row's state.
template <bool kExt>
__device__ __forceinline__ void fold_chunk(float (&v)[32], int col0, int V, RowState& st) {
  if (col0 + 32 > V) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j >= V) v[j] = -INFINITY;
  }
  float mx = v[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) mx = fmaxf(mx, v[j]);
  if (mx == -INFINITY) return;                 // the whole chunk is past the vocabulary
  float c2 = -INFINITY;                        // chunk's second largest (= mx on a tie)
  if constexpr (kExt) {
    int n_at_max = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      n_at_max += v[j] == mx ? 1 : 0;
      c2 = v[j] == mx ? c2 : fmaxf(c2, v[j]);
    }
    if (n_at_max > 1) c2 = mx;
  }
  if (mx > st.m) {                             // strict: earlier (lower) index wins ties
    int j0 = 31;
#pragma unroll
    for (int j = 31; j >= 0; --j)
      if (v[j] == mx) j0 = j;
    const float sc = ex2_approx((st.m - mx) * kLog2e);
    if constexpr (kExt) {
      // re-centre t on the new max: (z - mx) = (z - m) + (m - mx)
      if (st.s > 0.f) st.t = sc * (st.t + (st.m - mx) * st.s);
      st.m2 = fmaxf(st.m, c2);
    }
    st.s *= sc;
    st.m = mx;
    st.a = col0 + j0;
  } else if constexpr (kExt) {
    st.m2 = fmaxf(st.m2, mx);
  }
  const float mb = st.m * kLog2e;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
  if constexpr (kExt) {
    float t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float e0 = ex2_approx(fmaf(v[j + 0], kLog2e, -mb));
      const float e1 = ex2_approx(fmaf(v[j + 1], kLog2e, -mb));
      s0 += e0;
      s1 += e1;
      // past-the-vocabulary columns are -inf: e = 0, and 0 * (-inf) must not poison t
      t0 += e0 > 0.f ? e0 * (v[j + 0] - st.m) : 0.f;
      t1 += e1 > 0.f ? e1 * (v[j + 1] - st.m) : 0.f;
    }
    st.t += t0 + t1;
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      s0 += ex2_approx(fmaf(v[j + 0], kLog2e, -mb));
      s1 += ex2_approx(fmaf(v[j + 1], kLog2e, -mb));
      s2 += ex2_approx(fmaf(v[j + 2], kLog2e, -mb));
      s3 += ex2_approx(fmaf(v[j + 3], kLog2e, -mb));
    }
  }
  st.s += (s0 + s1) + (s2 + s3);
}

// Final values of a row state: tok, lse, conf (and entropy, margin).
__device__ __forceinline__ void state_finish(const RowState& st, int& tok, float& conf, float& lse,
                                             float& ent, float& margin) {
  tok = st.a;
  lse = st.m + logf(st.s);
  conf = 1.0f / st.s;
  ent = logf(st.s) - st.t / st.s;
  margin = (1.0f - ex2_approx((st.m2 - st.m) * kLog2e)) / st.s;
}

// Partials of one row per vocabulary split (structure of arrays).
struct Partials {
  float* m;
  float* s;
  int* a;
  float* t;    // extended mode only
  float* m2;   // extended mode only
};

// lse_merge of one row, as an accumulation: fold the partials found at base + j * stride for
// j = j0..j1-1 (ascending vocabulary ranges) into st:
//   m* = max_j m_j, s* = sum_j s_j exp(m_j - m*), a = a_j of the first j with m_j = m*,
//   t* = sum_j exp(m_j - m*) (t_j + (m_j - m*) s_j), m2* = the second largest of all m_j, m2_j.
// Then lse = m* + ln s* and conf = exp(m* - lse) = 1 / s* (state_finish).  Partials are read
// through L2 (other CTAs of the running kernel may have written them) in batches of 8 whose
// loads are all issued before any is used.
template <bool kExt>
__device__ __forceinline__ void merge_state(RowState& st, float m, float s, int a, float t, float m2) {
  if (m == -INFINITY) return;           // empty partial: nothing to add
  if (m > st.m) {                       // strict: the earlier split keeps a tie
    const float sc = ex2_approx((st.m - m) * kLog2e);
    if constexpr (kExt) {
      st.t = (st.s > 0.f ? sc * (st.t + (st.m - m) * st.s) : 0.f) + t;
      st.m2 = fmaxf(st.m, m2);
    }
    st.s = st.s * sc + s;
    st.m = m;
    st.a = a;
  } else {
    const float sc = ex2_approx((m - st.m) * kLog2e);
    if constexpr (kExt) {
      st.t += sc * (t + (m - st.m) * s);
      st.m2 = fmaxf(st.m2, m);
    }
    st.s += s * sc;
  }
}

template <bool kExt>
__device__ __forceinline__ void merge_acc(const Partials& P, long long base, long long stride,
                                          int j0, int j1, RowState& st) {
  constexpr int kBatch = 8;
  for (int jb = j0; jb < j1; jb += kBatch) {
    float mb[kBatch], sb[kBatch], tb[kBatch], m2b[kBatch];
    int ab[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      if (jb + q < j1) {
        const long long e = base + (jb + q) * stride;
        mb[q] = __ldcg(P.m + e);
        sb[q] = __ldcg(P.s + e);
        ab[q] = __ldcg(P.a + e);
        if constexpr (kExt) {
          tb[q] = __ldcg(P.t + e);
          m2b[q] = __ldcg(P.m2 + e);
        }
      } else {
        mb[q] = -INFINITY;
        sb[q] = 0.f;
        ab[q] = 0;
        tb[q] = 0.f;
        m2b[q] = -INFINITY;
      }
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) merge_state<kExt>(st, mb[q], sb[q], ab[q], tb[q], m2b[q]);
  }
}

// Merge n_split partials at base + j * stride (plain layout; test hook).
__device__ __forceinline__ void merge_row(const float* __restrict__ pm, const float* __restrict__ ps,
                                          const int* __restrict__ pa, long long base,
                                          long long stride, int n_split, int& tok, float& conf,
                                          float& lse) {
  RowState st;
  st.reset();
  Partials P{const_cast<float*>(pm), const_cast<float*>(ps), const_cast<int*>(pa), nullptr, nullptr};
  merge_acc<false>(P, base, stride, 0, n_split, st);
  float ent, margin;
  state_finish(st, tok, conf, lse, ent, margin);
}

template <int CG>
__device__ __forceinline__ void mma_issue(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc) {
  if constexpr (CG == 1) umma_bf16(d_tmem, a_desc, b_desc, idesc, acc);
  else umma_bf16_pair(d_tmem, a_desc, b_desc, idesc, acc);
}

// Arrive on barrier `bar` of every CTA of the group once the issued MMAs complete.
template <int CG>
__device__ __forceinline__ void mma_commit_all(uint32_t bar) {
  if constexpr (CG == 1) umma_commit(bar);
  else umma_commit_pair_both(bar);
}

// Results of the kernel (compacted row order).
struct Outputs {
  int* tok;
  float* conf;
  float* lse;
  float* entropy;   // extended mode: written when not null
  float* margin;    // extended mode: written when not null
  // Vocabulary-shard mode (raw.m not null): instead of the finished values, each row's
  // merged state over this launch's vocabulary (a shard of a larger one) is written, with
  // the argmax shifted by a_offset to a global token index; t and m2 in extended mode.
  Partials raw;
  int a_offset;
};

// The GEMM of one launch on a CTA (CG = 1) or on one CTA of a pair (CG = 2).  tmA / tmB
// point at the kernel's own __grid_constant__ tensor-map parameters (TMA needs their
// parameter-space address, never a copy).  waited: the kernel already passed
// griddepcontrol.wait (then the set-up below no longer overlaps the previous kernel).
template <int CG, int kMode>
__device__ __forceinline__ void lmhead_run(uint8_t* smem_raw, const CUtensorMap* tmA,
                                           const CUtensorMap* tmB, const int* __restrict__ count_ptr,
                                           bool waited, int n_cap, int V, int d, int gmax,
                                           const Partials& part, long long part_cap,
                                           int* __restrict__ unit_ctr, const Outputs& out,
                                           float* __restrict__ dbg_logits, int* __restrict__ status) {
  using C = Cfg<CG>;
  constexpr bool kDebugStore = kMode == kModeDebugStore;
  constexpr bool kExt = kMode == kModeStatsExt;
  Smem<CG> sm(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 1 ? 0u : cluster_ctarank();   // rank inside the CTA pair
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.tfull[b]), 1);
      mbar_init(smem_u32(&sm.tempty[b]), CG * kEpiWarps * 32);
    }
    mbar_init(smem_u32(sm.drain), 1);
    mbar_init(smem_u32(sm.epi_bar), kEpiWarps * 32);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmB);
  }
  if (warp == 1) {
    if constexpr (CG == 1) {
      tmem_alloc(smem_u32(sm.tmem_slot), kTmemCols);
      tmem_relinquish();
    } else {
      tmem_alloc_pair(smem_u32(sm.tmem_slot), kTmemCols);
      tmem_relinquish_pair();
    }
  }
  tc_fence_before();
  if constexpr (CG == 1) __syncthreads();
  else cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot;
  volatile int* abort_flag = sm.abort_flag;

  // everything above touched only this CTA's own resources; from here on the kernel reads
  // what the compaction and gather kernels wrote
  if (!waited) {
    pdl_wait();
    pdl_launch_dependents();
  }
  const int count = *count_ptr;
  const Plan pl = Plan::make(count < 0 ? 0 : (count > n_cap ? n_cap : count), V,
                             static_cast<int>(gridDim.x) / CG, gmax, C::BM);
  const int holder = static_cast<int>(blockIdx.x) / CG;
  const int KB = d / BK;
  // producer thread of the arming CTA: stages armed so far (bit s), and the phase parity of
  // the last arming of each stage (bit s), for the abort path's wait on loads in flight
  uint32_t armed_mask = 0, armed_parity = 0;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      // Each CTA stages its own 128 rows of Hm and 256/CG rows of W.  With CG = 2 the
      // completion is counted on the leader's full barrier (the address with the peer bit
      // cleared), which the leader arms for the bytes of both CTAs.
      uint32_t it = 0;
      // Pacing of the CTA-pair body (full groups): the holders of one stream read the same W
      // tiles, and W comes from HBM about once per group only while they stay within a few
      // tiles of each other; pairs drift apart over a long stream (measured: 182-421 GB of
      // DRAM reads per launch on B1 L131072 at r_m = 0.9 without pacing).  Each pair
      // publishes how many tiles it has started (the pairs of a stream start the same number
      // per full group); before a tile, a pair that is more than kPace tiles ahead of a
      // stream-mate waits for it (a lead of 2 tiles: measured faster than 1 on both B1
      // L131072 d4096, 88.2 vs 90.5 ms per GEMM, and B8 L8192 d2048, 14.5 vs 15.8 ms).  The mates' progress is read one tile ahead, so the check
      // costs the producer nothing unless it really has to wait; the slowest pair never
      // waits, so every wait ends (it is bounded all the same).
      constexpr int kPace = CG == 2 ? DLLM_PAIR_PACE : 0;
      constexpr int kMates = 40;                 // at least the pair body's group size
      int* const progress = unit_ctr + ((n_cap + 127) / 128 + 2);
      int started = 0;
      int seen[kMates];                          // the mates' progress as of the last tile
#pragma unroll
      for (int j = 0; j < kMates; ++j) seen[j] = 0;
      auto pace = [&](int m_tile) -> bool {
        if (kPace <= 0 || pl.ngroups < 2 || pl.rem || pl.gmax > kMates) return true;
        const int g = m_tile / pl.gmax;
        if (pl.group_size(g) != pl.gmax) return true;          // the last, smaller group
        if (rank == 0) st_relaxed_gpu(progress + holder, started);
        const int first = (holder / pl.gmax) * pl.gmax;        // the stream's first holder
        const int need = started - kPace;
        bool behind = false;
#pragma unroll
        for (int j = 0; j < kMates; ++j) behind |= j < pl.gmax && seen[j] < need;
        if (behind) {                                          // really ahead: fresh reads
          const unsigned long long t0 = globaltimer_ns();
          for (;;) {
            bool lag = false;
            for (int j = 0; j < pl.gmax; ++j) lag |= ld_relaxed_gpu(progress + first + j) < need;
            if (!lag) break;
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              atomicOr(status, kStatusTimeout);
              *abort_flag = 1;
              return false;
            }
            __nanosleep(128);
          }
        }
#pragma unroll
        for (int j = 0; j < kMates; ++j)                       // for the next tile's check
          if (j < pl.gmax) seen[j] = ld_relaxed_gpu(progress + first + j);
        return true;
      };
      auto load_tile = [&](int m_tile, int n) -> bool {
        if (!pace(m_tile)) return false;
        ++started;
        const int a_row = m_tile * C::BM + static_cast<int>(rank) * C::BM_CTA;
        const int b_row = n * BN + static_cast<int>(rank) * C::B_ROWS;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag, status)) return false;
#ifdef DLLM_FAULT_SKIP_STAGE
          // Failure-detection test builds only: this stage is never armed or loaded, so the
          // MMA issuer's bounded wait on it runs out and the kernel unwinds with a timeout.
          if (it == DLLM_FAULT_SKIP_STAGE) continue;
#endif
          const uint32_t fb = smem_u32(&sm.full[s]);
          armed_mask |= 1u << s;
          armed_parity = (armed_parity & ~(1u << s)) | (ph << s);
          if constexpr (CG == 1) {
            mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
            tma_load_2d(smem_u32(sm.a + s * C::A_BYTES), tmA, fb, kb * BK, a_row);
            tma_load_2d(smem_u32(sm.b + s * C::B_BYTES), tmB, fb, kb * BK, b_row);
          } else {
            if (leader) mbar_arrive_expect_tx(fb, CG * C::STAGE_BYTES);
            const uint32_t fb_leader = fb & kPeerBitMask;
            tma_load_2d_pair(smem_u32(sm.a + s * C::A_BYTES), tmA, fb_leader, kb * BK, a_row);
            tma_load_2d_pair(smem_u32(sm.b + s * C::B_BYTES), tmB, fb_leader, kb * BK, b_row);
          }
        }
        return true;
      };
      for_each_tile(pl, holder, load_tile);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------ MMA issuer --------------------------------
      uint32_t it = 0, tile = 0;
      auto mma_tile = [&](int, int) -> bool {
        const uint32_t buf = tile & 1u, tph = (tile >> 1) & 1u;
        if (!mbar_wait(smem_u32(&sm.tempty[buf]), tph ^ 1u, abort_flag, status)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1u;
          if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag, status)) return false;
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(sm.a + s * C::A_BYTES));
          const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sm.b + s * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < BK / UK; ++k) {
            // advance 16 bf16 = 32 bytes along K inside the swizzle atom
            mma_issue<CG>(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_all<CG>(smem_u32(&sm.empty[s]));   // stage free once these MMAs retire
        }
        mma_commit_all<CG>(smem_u32(&sm.tfull[buf]));     // accumulator ready for the epilogues
        ++tile;
        return true;
      };
      if (!for_each_tile(pl, holder, mma_tile)) {
        // Make sure no MMA is still writing TMEM before the columns are released.
        mma_commit_all<CG>(smem_u32(sm.drain));
        mbar_wait_drain(smem_u32(sm.drain), 0u, status);
      }
    }
  } else {
    // -------------------------------- epilogue ---------------------------------
    const int q = warp & 3;                      // TMEM lane quadrant of this warp
    const int row_in_cta = q * 32 + lane;
    const int row_in_tile = static_cast<int>(rank) * C::BM_CTA + row_in_cta;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t tile = 0, epi_phase = 0;
    bool ok = true;
    // all 128 epilogue threads meet; false (warp-uniform) if the CTA is aborting
    auto epi_sync = [&]() -> bool {
      mbar_arrive(smem_u32(sm.epi_bar));
      const bool got = mbar_wait(smem_u32(sm.epi_bar), epi_phase, abort_flag, status);
      epi_phase ^= 1u;
      return __all_sync(0xffffffffu, got);
    };
    // fold the next accumulator (vocabulary tile n of m-tile m_tile) into st
    auto consume = [&](int m_tile, int n, RowState& st) -> bool {
      const uint32_t buf = tile & 1u, tph = (tile >> 1) & 1u;
      // every lane waits; the vote reconverges the warp before the .sync.aligned loads and
      // makes the abort decision warp-uniform
      const bool got = DLLM_EPI_BACKOFF_NS > 0
                           ? mbar_wait_backoff(smem_u32(&sm.tfull[buf]), tph, abort_flag, status,
                                               DLLM_EPI_BACKOFF_NS)
                           : mbar_wait(smem_u32(&sm.tfull[buf]), tph, abort_flag, status);
      if (!__all_sync(0xffffffffu, got)) return false;
      tc_fence_after();
      const uint32_t taddr = lane_base + buf * BN;
      const int row = m_tile * C::BM + row_in_tile;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait();
        const int col0 = n * BN + c * 32;
        if constexpr (kDebugStore) {
          if (row < pl.count) {
            for (int j = 0; j < 32; ++j)
              if (col0 + j < V) dbg_logits[static_cast<size_t>(row) * V + col0 + j] = v[j];
          }
        } else {
          fold_chunk<kExt>(v, col0, V, st);
        }
      }
      tc_fence_before();
      // release the accumulator: the leader's MMA waits for the epilogues of both CTAs
      if constexpr (CG == 1) mbar_arrive(smem_u32(&sm.tempty[buf]));
      else mbar_arrive_cluster(smem_u32(&sm.tempty[buf]), 0u);
      ++tile;
      return true;
    };
    auto write_result = [&](int row, const RowState& st) {
      if (out.raw.m != nullptr) {
        out.raw.m[row] = st.m;
        out.raw.s[row] = st.s;
        out.raw.a[row] = st.a + out.a_offset;
        if constexpr (kExt) {
          if (out.raw.t) out.raw.t[row] = st.t;
          if (out.raw.m2) out.raw.m2[row] = st.m2;
        }
        return;
      }
      int t;
      float c, l, e, mg;
      state_finish(st, t, c, l, e, mg);
      out.tok[row] = t;
      out.conf[row] = c;
      out.lse[row] = l;
      if constexpr (kExt) {
        if (out.entropy) out.entropy[row] = e;
        if (out.margin) out.margin[row] = mg;
      }
    };
    auto write_partial = [&](long long e, const RowState& st) {
      if (e < part_cap) {
        part.m[e] = st.m;
        part.s[e] = st.s;
        part.a[e] = st.a;
        if constexpr (kExt) {
          part.t[e] = st.t;
          part.m2[e] = st.m2;
        }
      } else {
        atomicOr(status, kStatusBounds);             // cannot happen: workspace sized for it
      }
    };

    // A finished (m-tile, slot) state: the result itself when the m-tile has a single unit,
    // else a partial; the last of the m-tile's units to finish merges its rows.
    auto finish = [&](int g, const Unit& u, int m_local, int slot, const RowState& st) -> bool {
      const int m_tile = g * pl.gmax + m_local;
      const int row = m_tile * C::BM + row_in_tile;
      const bool valid = row < pl.count;
      int j_lo = 0, j_hi = -1;
      if (pl.rem) pl.leftovers_of(m_local, u.G, j_lo, j_hi);
      const int units = u.P + (j_hi >= j_lo ? j_hi - j_lo + 1 : 0);
      if (units == 1) {
        if (valid) write_result(row, st);
        return true;
      }
      if (valid) write_partial(pl.part_index(g, u.G, slot, m_local * C::BM + row_in_tile), st);
      // Writers fence before the counter increment; the last arriver fences after it and
      // reads the partials through L2.
      __threadfence();
      if (!epi_sync()) return false;
      if (threadIdx.x == 2 * 32) {
        const int old = atomicAdd(&unit_ctr[m_tile * CG + static_cast<int>(rank)], 1);
        *sm.last_flag = old == units - 1 ? 1 : 0;
      }
      if (!epi_sync()) return false;
      if (*sm.last_flag) {
        __threadfence();
        // The four epilogue warps split the m-tile's ordered partial slots (streams 0..P-1,
        // then remainder holders j_lo..j_hi): warp quarter q merges slots
        // [q * units / 4, (q + 1) * units / 4) for all 128 rows of this CTA, four rows per
        // lane, so that 4 x kMergeBatch partials per thread are in flight per L2 round trip
        // instead of kMergeBatch.  The quarters are then combined per row in slot order
        // through shared memory, which keeps vocabulary order (and so the tie rule).
        constexpr int kMergeBatch = kExt ? 4 : 8;
        const int row0 = m_tile * C::BM + static_cast<int>(rank) * C::BM_CTA;   // CTA's first row
        const int n_valid = pl.count - row0;
        const long long base0 = pl.part_index(g, u.G, 0, m_local * C::BM + static_cast<int>(rank) * C::BM_CTA);
        const long long stride = static_cast<long long>(u.G) * C::BM;
        const int s0 = q * units / 4, s1 = (q + 1) * units / 4;
        RowState acc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i].reset();
        for (int sb = s0; sb < s1; sb += kMergeBatch) {
          float mb[4][kMergeBatch], sv[4][kMergeBatch], tb[4][kMergeBatch], m2b[4][kMergeBatch];
          int ab[4][kMergeBatch];
#pragma unroll
          for (int j = 0; j < kMergeBatch; ++j) {
            const int sl = sb + j;
            const int slot = sl < u.P ? sl : u.P + j_lo + (sl - u.P);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = lane + 32 * i;
              if (sl < s1 && r < n_valid) {
                const long long e = base0 + slot * stride + r;
                mb[i][j] = __ldcg(part.m + e);
                sv[i][j] = __ldcg(part.s + e);
                ab[i][j] = __ldcg(part.a + e);
                if constexpr (kExt) {
                  tb[i][j] = __ldcg(part.t + e);
                  m2b[i][j] = __ldcg(part.m2 + e);
                }
              } else {
                mb[i][j] = -INFINITY;
                sv[i][j] = 0.f;
                ab[i][j] = 0;
                tb[i][j] = 0.f;
                m2b[i][j] = -INFINITY;
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < kMergeBatch; ++j)
              merge_state<kExt>(acc[i], mb[i][j], sv[i][j], ab[i][j], tb[i][j], m2b[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          auto& c = sm.comb[q * C::BM_CTA + lane + 32 * i];
          c.m = acc[i].m;
          c.s = acc[i].s;
          c.t = acc[i].t;
          c.m2 = acc[i].m2;
          c.a = acc[i].a;
        }
        if (!epi_sync()) return false;
        if (valid) {
          RowState fin;
          fin.reset();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const auto& c = sm.comb[k * C::BM_CTA + row_in_cta];
            merge_state<kExt>(fin, c.m, c.s, c.a, c.t, c.m2);
          }
          write_result(row, fin);
        }
      }
      return true;
    };

    for (int g = 0; g < pl.ngroups && ok; ++g) {
      Unit u;
      if (!unit_of(pl, g, holder, u)) continue;
      if (u.leftover) {
        // remainder tiles in m-major order: one running state, finished at each m-tile change
        int cur = -1;
        RowState st;
        st.reset();
        for (long long i = u.i0; i < u.i1 && ok; ++i) {
          const int m_local = static_cast<int>(i / pl.rr);
          const int n = u.P * pl.rb + static_cast<int>(i % pl.rr);
          if (m_local != cur) {
            if (cur >= 0 && !kDebugStore) ok = finish(g, u, cur, u.p, st);
            cur = m_local;
            st.reset();
          }
          if (ok && !consume(g * pl.gmax + m_local, n, st)) ok = false;
        }
        if (ok && cur >= 0 && !kDebugStore) ok = finish(g, u, cur, u.p, st);
      } else {
        RowState st;
        st.reset();
        for (int n = u.n0; n < u.n1 && ok; ++n)
          if (!consume(u.m_tile, n, st)) ok = false;
        if (ok && !kDebugStore) ok = finish(g, u, u.m_local, u.p, st);
      }
    }
  }

  tc_fence_before();
  if constexpr (CG == 1) __syncthreads();
  else cluster_sync();          // neither CTA leaves while its peer may still touch its smem
  // Every role has left its loop, so the abort flags no longer change; both CTAs of a pair
  // read both flags and take the same decision.
  bool aborted = *abort_flag != 0;
  if constexpr (CG == 2) {
    aborted = aborted || ld_shared_cluster_s32(smem_u32(sm.abort_flag), rank ^ 1u) != 0;
    cluster_sync();             // the peer's shared memory stays alive until both have read
  }
  if (aborted) {
    // Loads already issued must land before shared memory is released: wait for the last
    // armed phase of every stage (the arming CTA's barrier counts the loads of both CTAs of a
    // pair).  A phase that was armed but whose loads were never all issued (a CTA that
    // stopped first) holds the wait to the shared deadline, by which the issued loads have
    // long landed.
    if (warp == 0 && lane == 0 && (CG == 1 || leader)) {
      const unsigned long long deadline = globaltimer_ns() + kWaitLimitNs;
      for (int s = 0; s < C::kStages; ++s)
        if (armed_mask & (1u << s))
          if (!mbar_wait_until(smem_u32(&sm.full[s]), (armed_parity >> s) & 1u, deadline, status))
            break;
    }
    if constexpr (CG == 1) __syncthreads();
    else cluster_sync();
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (CG == 1) tmem_dealloc(tmem_base, kTmemCols);
    else tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// One GEMM variant, fixed at launch (CG = 2 needs a launch in clusters of two CTAs).  Its
// set-up (barriers, TMEM, tensor-map prefetch) runs before griddepcontrol.wait, overlapping
// the previous kernel on the stream.
template <int CG, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const int* __restrict__ count_ptr, int n_cap, int V, int d, int gmax,
              const Partials part, long long part_cap, int* __restrict__ unit_ctr,
              const Outputs out, float* __restrict__ dbg_logits, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  lmhead_run<CG, kMode>(smem_raw, &tmA, &tmB, count_ptr, false, n_cap, V, d, gmax, part, part_cap,
                        unit_ctr, out, dbg_logits, status);
}

// The variant chosen on the device from the masked count, which the host does not know:
// one m-tile of 128 rows or fewer runs on single CTAs (a pair would compute 128 empty
// rows), more on CTA pairs: per SM a third fewer bytes staged from L2 per flop, which under
// the 1 kW power cap is what sets the clock (measured on B1 L131072 at r_m = 0.9: the paced
// pair ran the GEMM in 89.8 ms at 1320 MHz where single CTAs took 99-100 ms at 1170 MHz).
// Launched in clusters of two CTAs with the shared memory of the larger variant; the count
// is read first, so the set-up follows griddepcontrol.wait.
constexpr int kSingleMaxRows = 128;
__host__ __device__ inline int auto_variant(int count) { return count > kSingleMaxRows ? 2 : 1; }
constexpr int kAutoSmemBytes = Cfg<1>::SMEM_BYTES > Cfg<2>::SMEM_BYTES ? Cfg<1>::SMEM_BYTES
                                                                        : Cfg<2>::SMEM_BYTES;

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_auto_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ CUtensorMap tmB2, const int* __restrict__ count_ptr,
                   int n_cap, int V, int d, const Partials part, long long part_cap,
                   int* __restrict__ unit_ctr, const Outputs out, float* __restrict__ dbg_logits,
                   int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  pdl_wait();
  pdl_launch_dependents();
  const int c = *count_ptr;
  if (auto_variant(c) == 2)
    lmhead_run<2, kMode>(smem_raw, &tmA, &tmB2, count_ptr, true, n_cap, V, d, Cfg<2>::kGroupM,
                         part, part_cap, unit_ctr, out, dbg_logits, status);
  else
    lmhead_run<1, kMode>(smem_raw, &tmA, &tmB1, count_ptr, true, n_cap, V, d, Cfg<1>::kGroupM,
                         part, part_cap, unit_ctr, out, dbg_logits, status);
}

}  // namespace lm
}  // namespace dllm
