// rank.cuh -- pieces of the exact k-th-largest search shared by the block-
// level ranker (select.cu) and the warp-level ranker (select_prefill.cu).
//
// Scores are ranked as orderable uint32 keys (orderable_key in common.cuh).
// A search pass splits the current "members" -- the keys inside one
// contiguous key interval -- into 256 bins by a function monotone in the key,
// so every bin is again an interval and equal keys share a bin; the bin that
// holds the wanted rank becomes the next members.
#pragma once

#include "common.cuh"

namespace sparda {

__device__ __forceinline__ float key_to_score(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// the member set after a pass: keys in [lo, hi] whose bin is `b`
struct Members {
  bool all;          // no pass yet: every key
  uint32_t lo, hi;
  bool by_score;     // bins linear in score (else linear in key)
  float base, inv;
  uint32_t b;
  __device__ __forceinline__ uint32_t bin(uint32_t u) const {
    const float x = by_score ? (key_to_score(u) - base) * inv : (float)(u - lo) * inv;
    return min(255u, __float2uint_rz(x));
  }
  __device__ __forceinline__ bool has(uint32_t u) const {
    return all || (u >= lo && u <= hi && bin(u) == b);
  }
};

// The bins of the next pass over members spanning keys [umin, umax]
// (umin < umax).  The first pass bins linearly in score value when that is
// well defined; later passes bin linearly in key space, which cuts the key
// range about 256-fold per pass.  Either way the smallest member lands in
// bin 0 and the largest in a bin >= 128, so each pass shrinks the range.
__device__ __forceinline__ Members make_bins(int pass, uint32_t umin, uint32_t umax) {
  Members nx{};
  nx.all = false;
  nx.lo = umin;
  nx.hi = umax;
  nx.by_score = false;
  if (pass == 0) {
    const float smin = key_to_score(umin), smax = key_to_score(umax);
    const float inv = 256.0f / (smax - smin);
    if (inv > 0.0f && inv < __int_as_float(0x7f800000)) {
      nx.by_score = true;
      nx.base = smin;
      nx.inv = inv;
    }
  }
  if (!nx.by_score) nx.inv = 256.0f / ((float)(umax - umin) + 1.0f);
  return nx;
}

}  // namespace sparda
