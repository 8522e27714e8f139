// Warp-cooperative lower_bound on an ascending int32 list: the first position
// p in [0, cnt) with idx[p] >= key, or cnt. Each round the 32 lanes probe 32
// evenly spaced entries at once and a ballot narrows the range 32-fold, so a
// list of 40k entries takes 4 dependent loads instead of 16. All 32 lanes must
// call it with the same arguments; every lane gets the result.
#pragma once

#include <stdint.h>

namespace tps {

__device__ __forceinline__ int64_t warp_lower_bound(const int32_t* __restrict__ idx, int64_t cnt, int64_t key,
                                                    int lane) {
  int64_t lo = 0, hi = cnt;                      // answer in [lo, hi]
  while (hi - lo > 32) {
    const int64_t step = (hi - lo + 31) >> 5;    // probes lo, lo+step, ..., all < hi
    const int64_t q = lo + static_cast<int64_t>(lane) * step;
    const bool less = q < hi && idx[q] < key;
    const int c = __popc(__ballot_sync(0xffffffffu, less));   // probes 0 .. c-1 are below key
    const int64_t nlo = c > 0 ? lo + static_cast<int64_t>(c - 1) * step + 1 : lo;
    const int64_t qc = lo + static_cast<int64_t>(c) * step;
    hi = qc < hi ? qc : hi;
    lo = nlo;
  }
  const int64_t q = lo + lane;
  const bool less = q < hi && idx[q] < key;
  return lo + __popc(__ballot_sync(0xffffffffu, less));
}

}  // namespace tps
