// compact.cuh - mask_compact: prefix-sum compaction of the masked positions, and the
// gather of the masked hidden rows into a dense matrix for the tensor-core GEMM.
//
// The Mosaic page (TL;DR, Abstract) computes logits at masked positions only; compaction
// turns the mask into the list of rows the LM head must see.
//
// Optional per-sequence windows [lo_b, hi_b) restrict the compaction to the masked positions
// of each sequence's current block.
//
// Launches over tiles of kCompactTile positions (one 16-byte vector per thread):
//   compact_count_kernel    tile t -> number of nonzero mask bytes in the tile
//   compact_scan_kernel     (more than kCompactDirectTiles tiles only) one CTA turns the
//                           counts into exclusive offsets, in place
//   compact_scatter_kernel  tile t -> its offset (read, or for at most kCompactDirectTiles
//                           tiles the sum of earlier tiles' counts reduced by the whole
//                           CTA), a block-wide exclusive scan of per-thread counts, then the
//                           ascending positions, seq_off and count.
#pragma once
#include "ptx.cuh"

namespace dllm {

constexpr int kCompactThreads = 512;
constexpr int kCompactVec = 16;                                   // bytes per thread
constexpr int kCompactTile = kCompactThreads * kCompactVec;       // 8192 positions
// Up to this many tiles each scatter CTA sums the earlier tiles' counts itself (at most 63
// loads); beyond it a scan launch computes every tile's offset once, so the total work stays
// linear in the number of tiles.
constexpr int kCompactDirectTiles = 64;
constexpr int kScanThreads = 1024;

// 0x80 in every byte of w that is nonzero, 0 elsewhere (no carries cross bytes because
// (b & 0x7F) + 0x7F <= 0xFE).
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t w) {
  return (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
}

// Loads the thread's 16 mask bytes starting at position p0 (bytes past n read as 0) and
// returns a 16-bit mask of nonzero positions (bit j = position p0 + j).
__device__ __forceinline__ uint32_t load_mask16(const uint8_t* __restrict__ M, long long p0,
                                                long long n) {
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if (p0 + kCompactVec <= n) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(M + p0));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if (p0 < n) {
    for (int j = 0; j < kCompactVec; ++j)
      if (p0 + j < n) w[j >> 2] |= static_cast<uint32_t>(M[p0 + j] != 0) << (8 * (j & 3));
  }
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t nz = nonzero_bytes(w[q]);
    // gather bit 7 of each byte into 4 consecutive bits
    const uint32_t b = ((nz >> 7) & 1u) | ((nz >> 14) & 2u) | ((nz >> 21) & 4u) | ((nz >> 28) & 8u);
    bits |= b << (4 * q);
  }
  return bits;
}

// Keeps the bits of `bits` (positions p0 + j, all < n) whose position lies inside its
// sequence's window: lo[b] <= l < hi[b] for position b * L + l.  Without windows (lo NULL)
// every bit is kept.  Semi-autoregressive decoding works on one block of each sequence at
// a time (Sparse-dLLM page, "Experiment"), so only the block's masked rows need logits.
__device__ __forceinline__ uint32_t window_filter(uint32_t bits, long long p0, int L,
                                                  const int* __restrict__ lo,
                                                  const int* __restrict__ hi) {
  if (lo == nullptr || bits == 0u) return bits;
  long long b = p0 / L;
  int l = static_cast<int>(p0 - b * L);
  int wl = __ldg(lo + b), wh = __ldg(hi + b);
  uint32_t keep = 0u;
  const int last = 31 - __clz(static_cast<int>(bits));            // highest set bit
  for (int j = 0; j <= last; ++j) {
    if (l >= wl && l < wh) keep |= 1u << j;
    if (++l == L && j < last) {          // position p0 + j + 1 <= p0 + last < n: b + 1 < B
      l = 0;
      ++b;
      wl = __ldg(lo + b);
      wh = __ldg(hi + b);
    }
  }
  return bits & keep;
}

// Block-wide sum of one int per thread (blockDim.x == kCompactThreads).
__device__ __forceinline__ int block_sum(int v, int* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int t = 0;
  if (warp == 0) {
    t = lane < kCompactThreads / 32 ? red[lane] : 0;
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

__global__ void __launch_bounds__(kCompactThreads)
compact_count_kernel(const uint8_t* __restrict__ M, long long n, int L, const int* __restrict__ win_lo,
                     const int* __restrict__ win_hi, int* __restrict__ tile_count) {
  __shared__ int red[33];
  pdl_wait();
  pdl_launch_dependents();
  const long long p0 = (static_cast<long long>(blockIdx.x) * kCompactThreads + threadIdx.x) * kCompactVec;
  const int c = __popc(window_filter(load_mask16(M, p0, n), p0, L, win_lo, win_hi));
  const int total = block_sum(c, red);
  if (threadIdx.x == 0) tile_count[blockIdx.x] = total;
}

// Exclusive prefix sum of the n tile counts, in place (one CTA): thread i sums a contiguous
// chunk, the chunk sums are scanned across the CTA, then each thread writes its chunk's
// offsets.
__global__ void __launch_bounds__(kScanThreads)
compact_scan_kernel(int* __restrict__ tile_count, int n) {
  __shared__ int warp_tot[kScanThreads / 32];
  pdl_wait();
  pdl_launch_dependents();
  const int per = (n + kScanThreads - 1) / kScanThreads;
  const int i0 = threadIdx.x * per;
  const int i1 = i0 + per < n ? i0 + per : n;
  int sum = 0;
  for (int i = i0; i < i1; ++i) sum += tile_count[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_tot[lane];               // kScanThreads / 32 == 32 warps
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - w;
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - sum;        // exclusive offset of this thread's chunk
  for (int i = i0; i < i1; ++i) {
    const int c = tile_count[i];
    tile_count[i] = run;
    run += c;
  }
}

__global__ void __launch_bounds__(kCompactThreads)
compact_scatter_kernel(const uint8_t* __restrict__ M, int B, int L, const int* __restrict__ win_lo,
                       const int* __restrict__ win_hi, const int* __restrict__ tile_count,
                       bool offsets, int* __restrict__ row_idx, int* __restrict__ seq_off,
                       int* __restrict__ count, int* __restrict__ status) {
  __shared__ int red[33];
  __shared__ int warp_excl[kCompactThreads / 32];
  pdl_wait();
  pdl_launch_dependents();
  const long long n = static_cast<long long>(B) * L;
  const int t = blockIdx.x;
  // offset of this tile = sum of the counts of tiles 0..t-1 (already scanned when `offsets`)
  int tile_base;
  if (offsets) {
    tile_base = tile_count[t];
  } else {
    int part = 0;
    for (int i = threadIdx.x; i < t; i += kCompactThreads) part += tile_count[i];
    tile_base = block_sum(part, red);
  }

  const long long p0 = (static_cast<long long>(t) * kCompactThreads + threadIdx.x) * kCompactVec;
  const uint32_t bits = window_filter(load_mask16(M, p0, n), p0, L, win_lo, win_hi);
  const int c = __popc(bits);
  // block-wide exclusive scan of c
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = c;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_excl[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kCompactThreads / 32 ? warp_excl[lane] : 0;
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kCompactThreads / 32) warp_excl[lane] = wi - w;
  }
  __syncthreads();
  const int base = tile_base + warp_excl[warp] + incl - c;

  // positions, ascending
  int o = base;
  uint32_t b = bits;
  if (b && (base < 0 || static_cast<long long>(base) + c > n)) {   // cannot happen: bad scan
    atomicOr(status, kStatusBounds);
    b = 0;
  }
  while (b) {
    const int j = __ffs(b) - 1;
    b &= b - 1;
    row_idx[o++] = static_cast<int>(p0 + j);
  }
  // seq_off[s] for every sequence whose first position s*L lies in [p0, p0 + 16)
  if (p0 < n) {
    const long long lim = p0 + kCompactVec < n ? p0 + kCompactVec : n;
    for (long long s = (p0 + L - 1) / L; s < B && s * L < lim; ++s) {
      const int before = __popc(bits & ((1u << static_cast<int>(s * L - p0)) - 1u));
      seq_off[s] = base + before;
    }
    if (lim == n) {             // the thread holding the last position writes the totals
      seq_off[B] = base + c;
      *count = base + c;
    }
  }
}

// Copy the masked rows H[row_idx[r]] (d bf16 each) into the dense matrix Hm[r] for
// r < count (one warp per row, 16-byte vectors), and zero n_zero ints at `zero`.  Hm holds
// n_cap rows: a larger count records kStatusCapacity and only the first n_cap rows are
// copied.
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kGatherThreads)
gather_rows_kernel(const uint16_t* __restrict__ H, const int* __restrict__ row_idx,
                   const int* __restrict__ count, long long n_pos, long long n_cap, int d,
                   uint16_t* __restrict__ Hm, int* __restrict__ zero, int n_zero,
                   int* __restrict__ status) {
  pdl_wait();
  pdl_launch_dependents();
  // also clear the GEMM's per-m-tile unit counters for this step
  for (int i = blockIdx.x * kGatherThreads + threadIdx.x; i < n_zero; i += gridDim.x * kGatherThreads)
    zero[i] = 0;
  int n = *count;
  if (n < 0 || n > n_pos) {                          // cannot happen: bad compaction
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, kStatusBounds);
    n = 0;
  } else if (n > n_cap) {                            // workspace sized for fewer rows
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, kStatusCapacity);
    n = static_cast<int>(n_cap);
  }
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kGatherThreads / 32);
  const int vec_per_row = d / 8;                     // uint4 = 8 bf16
  for (int r = blockIdx.x * (kGatherThreads / 32) + (threadIdx.x >> 5); r < n; r += warps) {
    const int p = row_idx[r];
    if (p < 0 || p >= n_pos) {
      if (lane == 0) atomicOr(status, kStatusBounds);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(H + static_cast<size_t>(p) * d);
    uint4* dst = reinterpret_cast<uint4*>(Hm + static_cast<size_t>(r) * d);
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
  }
}

}  // namespace dllm
