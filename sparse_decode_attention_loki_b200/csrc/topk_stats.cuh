// Agreement of two top-k selections: the Jaccard similarity |A n B| / |A u B|
// of the index sets of every (batch, KV head) row, the measure the Loki summary
// page reports between Loki's selection and the exact top-k ("Loki: Low-rank
// Keys for Efficient Sparse Attention", atlas.scime.ai, sections "Key results"
// and "Experimental setup").
//
// Both inputs are rows of k distinct token indices in ascending order, as
// loki_decode_attention writes them.  One CTA per row: each thread takes
// elements of A and binary-searches them in B; the matches are summed over the
// CTA.  J = c / (2k - c).
#pragma once

#include "common.cuh"

namespace loki {

struct JaccardArgs {
  const int32_t *a;  // [rows, k]
  const int32_t *b;  // [rows, k]
  float *out;        // [rows]
  int32_t k;
};

__global__ void __launch_bounds__(kThreads) topk_jaccard_kernel(const __grid_constant__ JaccardArgs p) {
  __shared__ uint32_t wtot[kWarps];
  const size_t row = blockIdx.x;
  const int32_t *a = p.a + row * (size_t)p.k;
  const int32_t *b = p.b + row * (size_t)p.k;
  uint32_t hits = 0u;
  for (int i = threadIdx.x; i < p.k; i += kThreads) {
    const int32_t x = __ldg(a + i);
    int lo = 0, hi = p.k;  // first position in b with b[pos] >= x
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(b + mid) < x) lo = mid + 1;
      else hi = mid;
    }
    hits += (lo < p.k && __ldg(b + lo) == x) ? 1u : 0u;
  }
  const uint32_t c = block_sum(hits, wtot);
  if (threadIdx.x == 0) p.out[row] = (float)c / (float)(2 * p.k - (int)c);
}

}  // namespace loki
