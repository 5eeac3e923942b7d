// Selected sets given as index lists (the shape tb_select writes: per query
// head, ascending token indices and a count) turned into the per-head
// bitmask the sparse attention reads.  One CTA per (b, h) row: it clears the
// row's words up to the sequence length, then sets one bit per listed index.
// Indices outside [0, len) are skipped and flag TB_DEV_ERR_INDEX; a count
// outside [0, idx_cap] flags it too and is clamped.
#pragma once

#include "common.cuh"

namespace tb {

struct IndexMaskParams {
  const int32_t* idx;    // [B][Hq][idx_cap]
  const int32_t* count;  // [B][Hq]
  uint32_t* mask;        // [B][Hq][mask_words]
  uint32_t* status;
  int Hq, idx_cap, mask_words;
  int lens[kMaxBatch];
};

constexpr int kIdxMaskThreads = 256;

// grid (Hq, B)
__global__ void __launch_bounds__(kIdxMaskThreads) index_mask_kernel(const IndexMaskParams p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int L = p.lens[b];
  const size_t row = (size_t)b * p.Hq + h;
  uint32_t* m = p.mask + row * p.mask_words;
  const int nw = (L + 31) >> 5;
  for (int w = tid; w < nw; w += kIdxMaskThreads) m[w] = 0u;
  __syncthreads();  // the row's words are cleared before any bit is set
  int n = p.count[row];
  if (n < 0 || n > p.idx_cap) {
    if (tid == 0) atomicOr(p.status, TB_DEV_ERR_INDEX);
    n = n < 0 ? 0 : p.idx_cap;
  }
  const int32_t* list = p.idx + row * p.idx_cap;
  bool bad = false;
  for (int i = tid; i < n; i += kIdxMaskThreads) {
    const int t = list[i];
    if (t < 0 || t >= L) {
      bad = true;
      continue;
    }
    atomicOr(&m[t >> 5], 1u << (t & 31));
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(p.status, TB_DEV_ERR_INDEX);
}

}  // namespace tb
