// Selection scores as integer sort keys, shared by the top-k (which expert a token picks)
// and the score-priority dispatch (which picks an expert keeps when it overflows), so that
// both take their decision on the same order.
#pragma once
#include <stdint.h>

namespace moe {

// Unsigned keys whose integer order is the float order: a larger key is a larger score.
// -0 and +0 map to one key (they compare equal as floats), a NaN maps to 1, below every
// number, and 0 is left for "not eligible".
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 1u;
  const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Priority of token t's pick of an expert whose selection score is `score`: the score's
// key above, the token index (inverted: lower token = higher priority) below.  Unique per
// (token, expert), so an expert's picks are totally ordered by it.
__device__ __forceinline__ uint64_t pick_priority(float score, int64_t t) {
  return (static_cast<uint64_t>(order_key(score)) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(t));
}

}  // namespace moe
