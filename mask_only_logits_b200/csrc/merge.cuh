// merge.cuh - lse_merge on plain-layout partials (test hook).  The decode step itself merges
// inside the GEMM epilogue (lm::merge_row in lmhead.cuh).
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

// Plain layout (index j * n_rows + i), used by the merge test hook.
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_plain_kernel(const float* __restrict__ pm, const float* __restrict__ ps,
                       const int* __restrict__ pa, int n_rows, int n_split, int* __restrict__ tok,
                       float* __restrict__ conf, float* __restrict__ lse) {
  for (int r = blockIdx.x * kMergeThreads + threadIdx.x; r < n_rows; r += gridDim.x * kMergeThreads) {
    int t;
    float c, l;
    lm::merge_row(pm, ps, pa, r, n_rows, n_split, t, c, l);
    tok[r] = t;
    conf[r] = c;
    lse[r] = l;
  }
}

}  // namespace dllm
