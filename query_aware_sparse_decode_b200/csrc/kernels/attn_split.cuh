// Split-K chunking of the sparse attention grid (host side).  Every entry
// point that launches the attention kernels uses this one rule, so equal
// inputs give equal splits and the same fp32 merge order.
#pragma once

#include "attn.cuh"

namespace tb {

// The grid is about two full waves of two CTAs per SM, or one wave when two
// would leave CTAs with short chunks (fewer than 3584 tokens: the list build,
// the ring's fill and the partial write then weigh more than the second
// wave's balance gains).  Chunks are multiples of 32 tokens (whole mask
// words), so that the splits fill the wave.  `groups` is B * Hkv.  Returns false when more than kMaxSplits splits would be needed.
inline bool attn_split(int num_sms, int groups, int maxL, int* chunk_out, int* nsplit_out) {
  const int L = maxL > 1 ? maxL : 1;
  int want = (4 * num_sms) / groups;
  want = want < 1 ? 1 : (want > kMaxSplits ? kMaxSplits : want);
  if ((L + want - 1) / want < 3584) {
    want = (2 * num_sms) / groups;
    want = want < 1 ? 1 : (want > kMaxSplits ? kMaxSplits : want);
  }
  int chunk = (L + want - 1) / want;
  chunk = (chunk + 31) / 32 * 32;
  const int n = (maxL + chunk - 1) / chunk;
  *chunk_out = chunk;
  *nsplit_out = n > 1 ? n : 1;
  return *nsplit_out <= kMaxSplits;
}

}  // namespace tb
