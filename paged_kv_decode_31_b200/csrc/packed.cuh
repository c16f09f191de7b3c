// packed.cuh -- index helpers for packed ("varlen") token layouts: sequence b
// owns the packed tokens cu[b] .. cu[b+1] - 1 (the cumulative query lengths
// of a packed multi-request forward, AstrAI "Select per-request final logits
// from cumulative query lengths").
#pragma once

#include <cstdint>

namespace pkv {

// Sequence of packed token tf: the largest b < batch with cu[b] <= tf (empty
// sequences share their start with the next one and are skipped by "largest").
__device__ __forceinline__ int seq_of_token(const int32_t *cu, int batch, int64_t tf) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= tf) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace pkv
