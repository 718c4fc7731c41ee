// merge.cuh - lse_merge: combine the per-vocabulary-split partials of each masked row into
// the predicted token, its log-sum-exp and its confidence.
//
// Partial j of a row holds m_j = max of its logits, s_j = sum exp(z - m_j) and a_j = the
// first argmax.  Splits are consecutive vocabulary ranges in ascending order, so
//   m* = max_j m_j,  s* = sum_j s_j exp(m_j - m*),  tok = a_j of the first j with m_j = m*,
//   lse = m* + ln s*,  conf = exp(m* - lse) = 1 / s*.
// (Mosaic page, Abstract: the mask-only logits kernel produces per-row predictions; the
// confidence is the largest softmax probability, the plainest reading of the confidence
// used by confidence-driven unmasking on the dLLM survey page, "Main Findings".)
#pragma once
#include "lmhead.cuh"

namespace dllm {

constexpr int kMergeThreads = 256;

// Merge n_split partials found at base + j * stride (j = 0..n_split-1).
__device__ __forceinline__ void merge_row(const float* __restrict__ pm, const float* __restrict__ ps,
                                          const int* __restrict__ pa, long long base,
                                          long long stride, int n_split, int& tok, float& conf,
                                          float& lse) {
  float m = -INFINITY, s = 0.f;
  int a = 0;
  for (int j = 0; j < n_split; ++j) {
    const long long e = base + j * stride;
    const float mj = pm[e];
    const float sj = ps[e];
    if (mj > m) {                    // strict: the earlier split keeps a tie
      s = s * ex2_approx((m - mj) * lm::kLog2e) + sj;
      m = mj;
      a = pa[e];
    } else {
      s += sj * ex2_approx((mj - m) * lm::kLog2e);
    }
  }
  tok = a;
  lse = m + logf(s);
  conf = 1.0f / s;
}

// Rows of the GEMM's unit schedule (see lm::Plan): row r belongs to group g = (r / BM) / gmax
// whose P streams each left one partial.
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(const int* __restrict__ count_ptr, int n_cap, int V, int ctas, int gmax,
                 const float* __restrict__ pm, const float* __restrict__ ps,
                 const int* __restrict__ pa, int* __restrict__ tok, float* __restrict__ conf,
                 float* __restrict__ lse) {
  int count = *count_ptr;
  count = count < 0 ? 0 : (count > n_cap ? n_cap : count);
  const lm::Plan pl = lm::Plan::make(count, V, ctas, gmax);
  for (int r = blockIdx.x * kMergeThreads + threadIdx.x; r < count; r += gridDim.x * kMergeThreads) {
    const int g = (r / lm::BM) / pl.gmax;
    const int G = pl.group_size(g);
    const int P = lm::Plan::streams(G, pl.ctas, pl.numN);
    const int r_in_group = r - g * pl.gmax * lm::BM;
    const long long base = pl.part_index(g, G, 0, r_in_group);
    int t;
    float c, l;
    merge_row(pm, ps, pa, base, static_cast<long long>(G) * lm::BM, P, t, c, l);
    tok[r] = t;
    conf[r] = c;
    lse[r] = l;
  }
}

// Plain layout (index j * n_rows + i), used by the merge test hook.
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_plain_kernel(const float* __restrict__ pm, const float* __restrict__ ps,
                       const int* __restrict__ pa, int n_rows, int n_split, int* __restrict__ tok,
                       float* __restrict__ conf, float* __restrict__ lse) {
  for (int r = blockIdx.x * kMergeThreads + threadIdx.x; r < n_rows; r += gridDim.x * kMergeThreads) {
    int t;
    float c, l;
    merge_row(pm, ps, pa, r, n_rows, n_split, t, c, l);
    tok[r] = t;
    conf[r] = c;
    lse[r] = l;
  }
}

}  // namespace dllm
