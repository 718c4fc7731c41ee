// lmhead.cuh - masked_lmhead: the mask-only LM head on the 5th-generation tensor cores with
// the softmax statistics fused into the epilogue (Mosaic page, TL;DR and Abstract: the
// mask-only logits kernel; the logits tensor of the masked rows is never written).
//
// C[i, v] = sum_k Hm[i, k] * W[v, k] for the compacted masked rows Hm (bf16, K-major) and
// the vocabulary projection W (bf16, K-major), fp32 accumulation in tensor memory.
//
// Persistent, warp-specialised kernel, one CTA per SM, 192 threads:
//   warp 0      TMA producer: 128x64 tile of Hm and 256x64 tile of W per stage
//               (128-byte swizzle) into a kStages-deep shared-memory ring
//   warp 1      allocates 512 TMEM columns; lane 0 issues tcgen05.mma (M=128, N=256,
//               K=16, four per stage) into one of two 128x256 fp32 accumulators and
//               commits stage releases / accumulator-full events to mbarriers
//   warps 2..5  epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (one row per thread) with
//               tcgen05.ld, keeps a running (max, sum exp(z - max), first argmax) per row
//               over the vocabulary tiles of its unit, then writes one partial per row
//
// Work decomposition.  A "unit" is (m-tile of 128 rows, contiguous range of vocabulary
// tiles).  m-tiles are taken in groups of up to `gmax`; inside a group of G m-tiles the CTAs
// are split into P = floor(ctas / G) vocabulary streams, CTA c handling m-tile c % G and
// stream c / G.  CTAs of one group therefore walk the same W tiles at the same time
// (each W tile is fetched from HBM about once per group and served to the other G-1 CTAs
// from L2) while the group's G Hm tiles stay resident in L2.  Per row, the partials of the
// P streams are merged by lse_merge.
#pragma once
#include "ptx.cuh"

namespace dllm {
namespace lm {

constexpr int BM = 128;                 // rows per tile (UMMA M)
constexpr int BN = 256;                 // vocabulary entries per tile (UMMA N)
constexpr int BK = 64;                  // K per stage: one 128-byte swizzle atom of bf16
constexpr int UK = 16;                  // K per tcgen05.mma (kind::f16)
constexpr int kStages = 4;
constexpr int A_BYTES = BM * BK * 2;    // 16 KiB
constexpr int B_BYTES = BN * BK * 2;    // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kTmemCols = 2 * BN;       // two accumulators
constexpr int kMaxCtas = 160;           // partial-buffer sizing bound (B200: 148 SMs)
constexpr int kGroupM = 37;             // m-tiles per L2 group (148 = 4 x 37)
constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + 256;

// Instruction descriptor, kind::f16: fp32 accumulator (bits 4-5 = 1), A and B bf16
// (bits 7-9 = 1, bits 10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                            (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);

constexpr float kLog2e = 1.4426950408889634f;

// The unit schedule, computed identically by the GEMM's three roles and by lse_merge.
struct Plan {
  int count, numM, numN, ctas, gmax, ngroups, P_full;

  __host__ __device__ static Plan make(int count, int V, int ctas, int gmax) {
    Plan p;
    p.count = count;
    p.numM = (count + BM - 1) / BM;
    p.numN = (V + BN - 1) / BN;
    p.ctas = ctas;
    p.gmax = gmax < ctas ? gmax : ctas;
    p.ngroups = (p.numM + p.gmax - 1) / p.gmax;
    p.P_full = streams(p.gmax, p.ctas, p.numN);
    return p;
  }
  __host__ __device__ static int streams(int G, int ctas, int numN) {
    int P = ctas / G;
    if (P > numN) P = numN;
    return P < 1 ? 1 : P;
  }
  __host__ __device__ int group_size(int g) const {
    return g == ngroups - 1 ? numM - g * gmax : gmax;
  }
  // Partial-buffer index of (group g of size G, stream p, row r within the group).
  __host__ __device__ long long part_index(int g, int G, int p, int r) const {
    return static_cast<long long>(g) * gmax * BM * P_full + static_cast<long long>(p) * G * BM + r;
  }
  // Number of partial entries written for this count (upper bound for sizing).
  __host__ __device__ long long part_entries() const {
    if (ngroups == 0) return 0;
    const int Gl = group_size(ngroups - 1);
    return part_index(ngroups - 1, Gl, 0, 0) +
           static_cast<long long>(Gl) * BM * streams(Gl, ctas, numN);
  }
};

// One unit of a CTA inside group g, or false if the CTA is idle in this group.
struct Unit {
  int m_tile, m_local, G, p, P, n0, n1;
};
__device__ __forceinline__ bool unit_of(const Plan& pl, int g, int cta, Unit& u) {
  u.G = pl.group_size(g);
  u.P = Plan::streams(u.G, pl.ctas, pl.numN);
  if (cta >= u.G * u.P) return false;
  u.m_local = cta % u.G;
  u.m_tile = g * pl.gmax + u.m_local;
  u.p = cta / u.G;
  u.n0 = static_cast<int>(static_cast<long long>(u.p) * pl.numN / u.P);
  u.n1 = static_cast<int>(static_cast<long long>(u.p + 1) * pl.numN / u.P);
  return true;
}

struct Smem {
  uint8_t* a;          // kStages x A_BYTES
  uint8_t* b;          // kStages x B_BYTES
  uint64_t* full;      // kStages
  uint64_t* empty;     // kStages
  uint64_t* tfull;     // 2
  uint64_t* tempty;    // 2
  uint64_t* drain;     // 1: MMA completion on the abort path
  uint32_t* tmem_slot;
  int* abort_flag;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.a = base;
  s.b = base + kStages * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.b + kStages * B_BYTES);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = bars + 2 * kStages + 2;
  s.drain = bars + 2 * kStages + 4;
  s.tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  s.abort_flag = reinterpret_cast<int*>(s.tmem_slot + 1);
  return s;
}

// Online (max, sum of exp(z - max), first argmax) over 32 consecutive logits.
__device__ __forceinline__ void fold_chunk(float (&v)[32], int col0, int V, float& run_m,
                                           float& run_s, int& run_a) {
  if (col0 + 32 > V) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j >= V) v[j] = -INFINITY;
  }
  float mx = v[0];
#pragma unroll
  for (int j = 1; j < 32; ++j) mx = fmaxf(mx, v[j]);
  if (mx == -INFINITY) return;                 // the whole chunk is past the vocabulary
  if (mx > run_m) {                            // strict: earlier (lower) index wins ties
    int j0 = 31;
#pragma unroll
    for (int j = 31; j >= 0; --j)
      if (v[j] == mx) j0 = j;
    run_s *= ex2_approx((run_m - mx) * kLog2e);
    run_m = mx;
    run_a = col0 + j0;
  }
  const float mb = run_m * kLog2e;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    s0 += ex2_approx(fmaf(v[j + 0], kLog2e, -mb));
    s1 += ex2_approx(fmaf(v[j + 1], kLog2e, -mb));
    s2 += ex2_approx(fmaf(v[j + 2], kLog2e, -mb));
    s3 += ex2_approx(fmaf(v[j + 3], kLog2e, -mb));
  }
  run_s += (s0 + s1) + (s2 + s3);
}

template <bool kDebugStore>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const int* __restrict__ count_ptr, int n_cap, int V, int d, int gmax,
              float* __restrict__ part_m, float* __restrict__ part_s, int* __restrict__ part_a,
              long long part_cap, float* __restrict__ dbg_logits, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.tfull[b]), 1);
      mbar_init(smem_u32(&sm.tempty[b]), kEpiWarps * 32);
    }
    mbar_init(smem_u32(sm.drain), 1);
    *sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot;
  volatile int* abort_flag = sm.abort_flag;

  const int count = *count_ptr;
  const Plan pl = Plan::make(count < 0 ? 0 : (count > n_cap ? n_cap : count), V, gridDim.x, gmax);
  const int cta = blockIdx.x;
  const int KB = d / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      uint32_t it = 0;
      bool ok = true;
      for (int g = 0; g < pl.ngroups && ok; ++g) {
        Unit u;
        if (!unit_of(pl, g, cta, u)) continue;
        for (int n = u.n0; n < u.n1 && ok; ++n) {
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&sm.empty[s]), ph ^ 1u, abort_flag, status)) { ok = false; break; }
            const uint32_t fb = smem_u32(&sm.full[s]);
            mbar_arrive_expect_tx(fb, STAGE_BYTES);
            tma_load_2d(smem_u32(sm.a + s * A_BYTES), &tmA, fb, kb * BK, u.m_tile * BM);
            tma_load_2d(smem_u32(sm.b + s * B_BYTES), &tmB, fb, kb * BK, n * BN);
          }
        }
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory goes away.
        const uint32_t first = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u;
        for (uint32_t j = first; j < it; ++j)
          mbar_wait_drain(smem_u32(&sm.full[j % kStages]), (j / kStages) & 1u, status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------ MMA issuer --------------------------------
      uint32_t it = 0, tile = 0;
      bool ok = true;
      for (int g = 0; g < pl.ngroups && ok; ++g) {
        Unit u;
        if (!unit_of(pl, g, cta, u)) continue;
        for (int n = u.n0; n < u.n1 && ok; ++n, ++tile) {
          const uint32_t buf = tile & 1u, tph = (tile >> 1) & 1u;
          if (!mbar_wait(smem_u32(&sm.tempty[buf]), tph ^ 1u, abort_flag, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * BN;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&sm.full[s]), ph, abort_flag, status)) { ok = false; break; }
            tc_fence_after();
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(sm.a + s * A_BYTES));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(sm.b + s * B_BYTES));
#pragma unroll
            for (int k = 0; k < BK / UK; ++k) {
              // advance 16 bf16 = 32 bytes along K inside the swizzle atom
              umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(&sm.empty[s]));     // stage free once these MMAs retire
          }
          if (!ok) break;
          umma_commit(smem_u32(&sm.tfull[buf]));     // accumulator ready for the epilogue
        }
      }
      if (!ok) {
        // Make sure no MMA is still writing TMEM before the columns are released.
        umma_commit(smem_u32(sm.drain));
        mbar_wait_drain(smem_u32(sm.drain), 0u, status);
      }
    }
  } else {
    // -------------------------------- epilogue ---------------------------------
    const int q = warp & 3;                      // TMEM lane quadrant of this warp
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t tile = 0;
    bool ok = true;
    for (int g = 0; g < pl.ngroups && ok; ++g) {
      Unit u;
      if (!unit_of(pl, g, cta, u)) continue;
      const int row = u.m_tile * BM + row_in_tile;
      float run_m = -INFINITY, run_s = 0.f;
      int run_a = 0;
      for (int n = u.n0; n < u.n1; ++n, ++tile) {
        const uint32_t buf = tile & 1u, tph = (tile >> 1) & 1u;
        // every lane waits; the vote reconverges the warp before the .sync.aligned loads and
        // makes the abort decision warp-uniform
        const bool got = mbar_wait(smem_u32(&sm.tfull[buf]), tph, abort_flag, status);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = lane_base + buf * BN;
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
            fold_chunk(v, col0, V, run_m, run_s, run_a);
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.tempty[buf]));
      }
      if (!ok) break;
      if (!kDebugStore && row < pl.count) {
        const long long e = pl.part_index(g, u.G, u.p, u.m_local * BM + row_in_tile);
        if (e < part_cap) {
          part_m[e] = run_m;
          part_s[e] = run_s;
          part_a[e] = run_a;
        } else {
          atomicOr(status, kStatusBounds);           // cannot happen: workspace sized for it
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace lm
}  // namespace dllm
