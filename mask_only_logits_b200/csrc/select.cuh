// select.cuh - select_unmask: per-sequence top-k of the confidences (confidence-driven
// unmasking, dLLM inference survey page, "Main Findings"), optionally restricted to a
// window [lo, hi) of positions (the current semi-autoregressive block: Sparse-dLLM page,
// "Experiment", block-wise decoding needs the current block only).
//
// Threshold-based parallel unmasking uses the same kernel (decoding thresholds, Dynamic-dLLM
// abstract on the dLLM pages): with a threshold, the number taken from a sequence is
// min(k, max(min(min_sel, n), #candidates with score >= threshold)); without one, min(k, n).
// In ascending order (e.g. entropy: lower is better) every comparison is reversed.
//
// One CTA of 1024 threads per sequence.  Key of a candidate in compacted row r:
//     (order-preserving bits of score[r]) << 32 | ~r
// Order-preserving bits: a float's IEEE bits with the sign bit flipped, or all bits flipped
// for negative values, compare as unsigned integers like the floats (scores may be negative,
// e.g. minus an entropy).  Within a sequence r ascends with the position, so ~r puts the
// lower position first among equal scores.
// Steps:
//   1. candidate range: rows of the sequence whose position lies in the window (one pass:
//      the window's rows are contiguous because row_idx ascends); with a threshold, the
//      number of candidates at or above it, hence k_eff, the number to take
//   2. if there are more than k_eff candidates, a 4-pass radix select (8 bits per pass) over
//      the 32 key bits finds T, the k_eff-th largest key, and how many of the candidates
//      equal to T are needed
//   3. one ordered pass collects every candidate above T and the first needed ones equal
//      to T (block-wide ballot scan keeps them in row order)
//   4. bitonic sort of the (at most k_eff) keys, descending; write positions, tokens, scores.
// Up to kSelRankMax candidates (e.g. one 32-token block) skip steps 2-4: keys are distinct,
// so the number of candidates whose key is larger is a candidate's place in the sorted
// output, and each thread writes its own candidate there if that place is below k_eff
// (about n^2 / 32 cycles, against ~25 CTA-wide barriers for steps 2-4).
#pragma once
#include "ptx.cuh"

namespace dllm {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxK = 1024;
constexpr int kSelStage = 4096;     // up to this many candidates: keys staged in shared memory
constexpr int kSelRankMax = 256;    // up to this many: output place by rank, no select or sort
// Passes over candidates read kSelUnroll keys per thread (rows base + j * kSelThreads + tid)
// before using any, so that a pass over a long sequence (e.g. 117961 candidates: 15 chunks
// instead of 116 dependent loads per thread) is not bound by one L2 round trip per key.
constexpr int kSelUnroll = 8;
static_assert(kSelRankMax <= kSelThreads && kSelRankMax <= kSelStage, "one staged key per thread");

// Float -> unsigned with the same order (for non-NaN values).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ unsigned long long sel_key(uint32_t okey, int r) {
  return (static_cast<unsigned long long>(okey) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(r));
}

__global__ void __launch_bounds__(kSelThreads, 1)
select_unmask_kernel(const float* __restrict__ conf, const int* __restrict__ row_idx,
                     const int* __restrict__ seq_off, int n_pos, int L, int k,
                     bool use_threshold, float threshold, int min_sel, bool ascending,
                     const int* __restrict__ win_lo, const int* __restrict__ win_hi,
                     const int* __restrict__ tok, int* __restrict__ idx, int* __restrict__ n_sel,
                     int* __restrict__ tok_sel, float* __restrict__ conf_sel) {
  __shared__ unsigned long long keys[kSelMaxK];
  __shared__ uint32_t skey[kSelStage];
  __shared__ unsigned int hist[256];
  __shared__ int sh_lo, sh_hi, sh_n, sh_digit, sh_krem, sh_taken, sh_q;
  __shared__ int blk_cnt[kSelUnroll * 32];      // collect: equal keys per (block of rows, warp)
  __shared__ int blk_tot[kSelUnroll];

  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // key of a score: larger key = better (ascending order: smaller score = better)
  const uint32_t flip = ascending ? 0xFFFFFFFFu : 0u;
  auto okey = [&](float f) -> uint32_t { return ordered_bits(f) ^ flip; };
  // compacted rows of sequence b (clamped: seq_off comes from the device)
  const int r0 = max(0, min(seq_off[b], n_pos));
  const int r1 = max(r0, min(seq_off[b + 1], n_pos));
  const long long seq_base = static_cast<long long>(b) * L;

  // 1. candidate range [c0, c1)
  int c0 = r0, c1 = r1;
  if (win_lo != nullptr) {
    const long long lo = seq_base + win_lo[b], hi = seq_base + win_hi[b];
    if (tid == 0) { sh_lo = r1; sh_hi = r0; }
    __syncthreads();
    int my_lo = r1, my_hi = r0;
    for (int r = r0 + tid; r < r1; r += kSelThreads) {
      const long long p = row_idx[r];
      if (p >= lo && p < hi) {
        my_lo = min(my_lo, r);
        my_hi = max(my_hi, r + 1);
      }
    }
    atomicMin(&sh_lo, my_lo);
    atomicMax(&sh_hi, my_hi);
    __syncthreads();
    c0 = sh_lo;
    c1 = sh_hi > sh_lo ? sh_hi : sh_lo;
  }
  const int n = c1 - c0;
  // small candidate sets: read the scores once and keep their keys in shared memory
  const bool staged = n <= kSelStage;
  if (staged) {
    for (int r = c0 + tid; r < c1; r += kSelThreads) skey[r - c0] = okey(conf[r]);
    __syncthreads();
  }
  auto key_of = [&](int r) -> uint32_t { return staged ? skey[r - c0] : okey(conf[r]); };
  int k_eff = n < k ? n : k;
  if (use_threshold) {
    if (tid == 0) sh_q = 0;
    __syncthreads();
    const uint32_t tq = okey(threshold);
    int mine = 0;
#pragma unroll 8
    for (int r = c0 + tid; r < c1; r += kSelThreads) mine += key_of(r) >= tq ? 1 : 0;
    for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
    if (lane == 0 && mine) atomicAdd(&sh_q, mine);
    __syncthreads();
    const int floor_n = min_sel < n ? min_sel : n;
    const int want = sh_q > floor_n ? sh_q : floor_n;
    k_eff = want < k ? want : k;
  }
  const int nsel = k_eff;

  if (n <= kSelRankMax) {            // uniform over the CTA: every thread returns here
    if (tid < n) {
      const uint32_t mine = skey[tid];
      int place = 0;                   // candidates ahead: larger key, or equal and lower row
      for (int j = 0; j < n; ++j) {
        const uint32_t other = skey[j];
        place += (other > mine || (other == mine && j < tid)) ? 1 : 0;
      }
      if (place < nsel) {
        const int r = c0 + tid;
        const size_t o = static_cast<size_t>(b) * k + place;
        idx[o] = static_cast<int>(row_idx[r] - seq_base);
        if (tok_sel) tok_sel[o] = tok[r];
        if (conf_sel) conf_sel[o] = conf[r];
      }
    }
    for (int j = nsel + tid; j < k; j += kSelThreads) {
      const size_t o = static_cast<size_t>(b) * k + j;
      idx[o] = -1;
      if (tok_sel) tok_sel[o] = -1;
      if (conf_sel) conf_sel[o] = 0.f;
    }
    if (tid == 0) n_sel[b] = nsel;
    return;
  }

  if (tid == 0) sh_n = 0;
  __syncthreads();

  if (n <= k_eff) {
    // 2'. every candidate is selected
    for (int r = c0 + tid; r < c1; r += kSelThreads) keys[r - c0] = sel_key(key_of(r), r);
  } else if (k_eff > 0) {
    // 2. radix select of the k_eff-th largest key.  Candidates not staged in shared memory
    // use that buffer for one 16-bit histogram per warp instead: confidences crowd into a
    // few bins, and one shared counter per bin had all 32 warps adding to the same words
    // (a warp sees at most 32 keys per 1024 candidates a pass: 32768 at 2^20 candidates,
    // within 16 bits).
    uint32_t prefix = 0, pmask = 0;
    int krem = k_eff;
    const bool warp_hist = !staged && n <= (1 << 20);
    uint16_t (*whist)[256] = reinterpret_cast<uint16_t (*)[256]>(skey);
    static_assert(sizeof(skey) >= 32 * 256 * sizeof(uint16_t), "per-warp histograms fit");
    for (int shift = 24; shift >= 0; shift -= 8) {
      if (warp_hist)
        for (int i = tid; i < 32 * 256 / 2; i += kSelThreads) skey[i] = 0u;
      else
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      // warp-aggregated histogram: confidences crowd into few bins (most share their top
      // bits), so lanes with the same bin add their count once
      for (int base = c0; base < c1; base += kSelThreads * kSelUnroll) {
        uint32_t u[kSelUnroll];
#pragma unroll
        for (int j = 0; j < kSelUnroll; ++j) {
          const int r = base + j * kSelThreads + tid;
          u[j] = r < c1 ? key_of(r) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kSelUnroll; ++j) {
          const int r = base + j * kSelThreads + tid;
          uint32_t bin = 0xFFFFFFFFu;
          if (r < c1 && (u[j] & pmask) == prefix) bin = (u[j] >> shift) & 255u;
          const unsigned peers = __match_any_sync(0xffffffffu, bin);
          if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) {
            if (warp_hist)
              whist[warp][bin] = static_cast<uint16_t>(whist[warp][bin] + __popc(peers));
            else
              atomicAdd(&hist[bin], __popc(peers));
          }
        }
      }
      __syncthreads();
      if (warp_hist) {
        for (int i = tid; i < 256; i += kSelThreads) {
          unsigned tot = 0;
#pragma unroll 8
          for (int w = 0; w < 32; ++w) tot += whist[w][i];
          hist[i] = tot;
        }
        __syncthreads();
      }
      if (warp == 0) {
        // lane l owns bins 255-8l down to 248-8l (descending order of digits)
        int own = 0;
        for (int j = 0; j < 8; ++j) own += hist[255 - 8 * lane - j];
        int incl = own;
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int excl = incl - own;
        if (excl < krem && krem <= incl) {
          int cum = excl;
          for (int j = 0; j < 8; ++j) {
            const int bin = 255 - 8 * lane - j;
            const int h = hist[bin];
            if (cum + h >= krem) { sh_digit = bin; sh_krem = krem - cum; break; }
            cum += h;
          }
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sh_digit) << shift;
      pmask |= 255u << shift;
      krem = sh_krem;
      __syncthreads();
    }
    // 3. collect: all above T, and the first krem equal to T in row order.  Rows are taken
    // kSelUnroll blocks of kSelThreads at a time; the equal keys are counted per (block,
    // warp) and scanned in that order, which is row order, with four barriers per chunk.
    const uint32_t T = prefix;
    if (tid == 0) sh_taken = 0;
    __syncthreads();
    for (int base = c0; base < c1; base += kSelThreads * kSelUnroll) {
      uint32_t uu[kSelUnroll];
      unsigned bal[kSelUnroll];
#pragma unroll
      for (int j = 0; j < kSelUnroll; ++j) {
        const int r = base + j * kSelThreads + tid;
        uu[j] = r < c1 ? key_of(r) : 0u;
      }
#pragma unroll
      for (int j = 0; j < kSelUnroll; ++j) {
        const int r = base + j * kSelThreads + tid;
        if (r < c1 && uu[j] > T) keys[atomicAdd(&sh_n, 1)] = sel_key(uu[j], r);
        bal[j] = __ballot_sync(0xffffffffu, r < c1 && uu[j] == T);
        if (lane == 0) blk_cnt[j * 32 + warp] = __popc(bal[j]);
      }
      __syncthreads();
      // exclusive scan of blk_cnt in (block, warp) order: warps 0..kSelUnroll-1 scan one
      // block each, then each block adds the totals of the blocks before it
      int v = 0, incl = 0;
      if (tid < kSelUnroll * 32) {
        v = blk_cnt[tid];
        incl = v;
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) blk_tot[warp] = incl;
      }
      __syncthreads();
      if (tid < kSelUnroll * 32) {
        int before_blocks = sh_taken;
        for (int b2 = 0; b2 < warp; ++b2) before_blocks += blk_tot[b2];
        blk_cnt[tid] = before_blocks + incl - v;
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kSelUnroll; ++j) {
        const int r = base + j * kSelThreads + tid;
        if (r < c1 && uu[j] == T) {
          const int before = blk_cnt[j * 32 + warp] + __popc(bal[j] & ((1u << lane) - 1u));
          if (before < krem) keys[atomicAdd(&sh_n, 1)] = sel_key(uu[j], r);
        }
      }
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int b2 = 0; b2 < kSelUnroll; ++b2) tot += blk_tot[b2];
        sh_taken += tot;
      }
    }
  }
  __syncthreads();

  // 4. bitonic sort of nsel keys, descending (padding keys are 0 and sink to the end)
  int P2 = 1;
  while (P2 < nsel) P2 <<= 1;
  for (int i = nsel + tid; i < P2; i += kSelThreads) keys[i] = 0ull;
  __syncthreads();
  for (int size = 2; size <= P2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < P2; i += kSelThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = keys[i], c = keys[j];
          if (desc ? (a < c) : (a > c)) { keys[i] = c; keys[j] = a; }
        }
      }
      __syncthreads();
    }
  }

  // 5. outputs
  for (int j = tid; j < k; j += kSelThreads) {
    const size_t o = static_cast<size_t>(b) * k + j;
    if (j < nsel) {
      const unsigned long long key = keys[j];
      const int r = static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffull));
      idx[o] = static_cast<int>(row_idx[r] - seq_base);
      if (tok_sel) tok_sel[o] = tok[r];
      if (conf_sel) conf_sel[o] = conf[r];
    } else {
      idx[o] = -1;
      if (tok_sel) tok_sel[o] = -1;
      if (conf_sel) conf_sel[o] = 0.f;
    }
  }
  if (tid == 0) n_sel[b] = nsel;
}

}  // namespace dllm
