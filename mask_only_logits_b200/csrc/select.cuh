// select.cuh - select_unmask: per-sequence top-k of the confidences (confidence-driven
// unmasking, dLLM inference survey page, "Main Findings"), optionally restricted to a
// window [lo, hi) of positions (the current semi-autoregressive block: Sparse-dLLM page,
// "Experiment", block-wise decoding needs the current block only).
//
// One CTA of 1024 threads per sequence.  Key of a candidate in compacted row r:
//     (float bits of conf[r]) << 32 | ~r
// Confidences are positive, so their IEEE bits order like the values; within a sequence r
// ascends with the position, so ~r puts the lower position first among equal confidences.
// Steps:
//   1. candidate range: rows of the sequence whose position lies in the window (one pass:
//      the window's rows are contiguous because row_idx ascends)
//   2. if there are more than k candidates, a 4-pass radix select (8 bits per pass) over
//      the 32 confidence bits finds T, the k-th largest confidence, and how many of the
//      candidates equal to T are needed
//   3. one ordered pass collects every candidate above T and the first needed ones equal
//      to T (block-wide ballot scan keeps them in row order)
//   4. bitonic sort of the (at most k) keys, descending; write positions, tokens, confs.
#pragma once
#include "ptx.cuh"

namespace dllm {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxK = 1024;

__device__ __forceinline__ unsigned long long sel_key(float c, int r) {
  return (static_cast<unsigned long long>(__float_as_uint(c)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(r));
}

__global__ void __launch_bounds__(kSelThreads)
select_unmask_kernel(const float* __restrict__ conf, const int* __restrict__ row_idx,
                     const int* __restrict__ seq_off, int n_pos, int L, int k,
                     const int* __restrict__ win_lo, const int* __restrict__ win_hi,
                     const int* __restrict__ tok, int* __restrict__ idx, int* __restrict__ n_sel,
                     int* __restrict__ tok_sel, float* __restrict__ conf_sel) {
  __shared__ unsigned long long keys[kSelMaxK];
  __shared__ unsigned int hist[256];
  __shared__ int sh_lo, sh_hi, sh_n, sh_digit, sh_krem, sh_taken;
  __shared__ int warp_cnt[32];

  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  const int nsel = n < k ? n : k;

  if (tid == 0) sh_n = 0;
  __syncthreads();

  if (n <= k) {
    // 2'. every candidate is selected
    for (int r = c0 + tid; r < c1; r += kSelThreads) keys[r - c0] = sel_key(conf[r], r);
  } else {
    // 2. radix select of the k-th largest confidence bits
    uint32_t prefix = 0, pmask = 0;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      // warp-aggregated histogram: confidences crowd into few bins (most share their top
      // bits), so lanes with the same bin add their count once
      for (int base = c0; base < c1; base += kSelThreads) {
        const int r = base + tid;
        uint32_t bin = 0xFFFFFFFFu;
        if (r < c1) {
          const uint32_t u = __float_as_uint(conf[r]);
          if ((u & pmask) == prefix) bin = (u >> shift) & 255u;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      __syncthreads();
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
    // 3. collect: all above T, and the first krem equal to T in row order
    const uint32_t T = prefix;
    if (tid == 0) sh_taken = 0;
    __syncthreads();
    for (int base = c0; base < c1; base += kSelThreads) {
      const int r = base + tid;
      uint32_t u = 0;
      if (r < c1) u = __float_as_uint(conf[r]);
      const bool gt = r < c1 && u > T;
      const bool eq = r < c1 && u == T;
      if (gt) keys[atomicAdd(&sh_n, 1)] = sel_key(__uint_as_float(u), r);
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) warp_cnt[warp] = __popc(bal);
      __syncthreads();
      int before = sh_taken;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w];
      before += __popc(bal & ((1u << lane) - 1u));
      if (eq && before < krem) keys[atomicAdd(&sh_n, 1)] = sel_key(__uint_as_float(u), r);
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < kSelThreads / 32; ++w) tot += warp_cnt[w];
        sh_taken += tot;
      }
      __syncthreads();
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
      if (conf_sel) conf_sel[o] = __uint_as_float(static_cast<uint32_t>(key >> 32));
    } else {
      idx[o] = -1;
      if (tok_sel) tok_sel[o] = -1;
      if (conf_sel) conf_sel[o] = 0.f;
    }
  }
  if (tid == 0) n_sel[b] = nsel;
}

}  // namespace dllm
