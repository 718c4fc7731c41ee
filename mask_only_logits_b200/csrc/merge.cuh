// merge.cuh - lse_merge as a kernel of its own: over the partials of vocabulary shards (one
// per GPU of a vocabulary-parallel LM head, gathered after the GEMM), and on plain-layout
// partials (test hook).  A single-GPU decode step merges inside the GEMM epilogue instead
// (lm::merge_acc in lmhead.cuh).
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

// Shard layout: split j of row i at j * split_stride + i, for rows i < *count (clamped to
// n_cap); splits in ascending vocabulary order.  Extended mode also merges t and m2 and
// writes entropy and / or margin where those outputs are given.
template <bool kExt>
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(lm::Partials part, long long split_stride, int n_split,
                 const int* __restrict__ count, int n_cap, lm::Outputs out) {
  pdl_wait();
  pdl_launch_dependents();
  int n = *count;
  n = n < 0 ? 0 : (n > n_cap ? n_cap : n);
  for (int r = blockIdx.x * kMergeThreads + threadIdx.x; r < n; r += gridDim.x * kMergeThreads) {
    lm::RowState st;
    st.reset();
    lm::merge_acc<kExt>(part, r, split_stride, 0, n_split, st);
    int t;
    float c, l, e, mg;
    lm::state_finish(st, t, c, l, e, mg);
    out.tok[r] = t;
    out.conf[r] = c;
    out.lse[r] = l;
    if constexpr (kExt) {
      if (out.entropy) out.entropy[r] = e;
      if (out.margin) out.margin[r] = mg;
    }
  }
}

}  // namespace dllm
