// order_key.cuh -- scores as order-preserving unsigned keys.
//
// order_key maps a float to a 32-bit key whose unsigned order is the float's
// order (larger score -> larger key; -0 and +0 map to one key).  key_value is
// its inverse (a key maps back to the float it came from, +0 for both
// zeros).  The max aggregation merges the observation groups' maxima as keys
// (an unsigned max in L2), and the top-K select ranks keys.
#pragma once
#include <cstdint>

namespace bkv {

__device__ __forceinline__ uint32_t order_key(float f) {
  // f + 0 is +0 for f = -0 (round to nearest) and f otherwise; then the
  // sign's arithmetic shift flips all bits of a negative and only the sign
  // bit of a positive
  const uint32_t u = __float_as_uint(f + 0.f);
  return u ^ (static_cast<uint32_t>(static_cast<int32_t>(u) >> 31) | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  // a key with its top bit set came from a non-negative float (flip the sign
  // bit back); otherwise from a negative one (flip every bit back)
  return __uint_as_float(k ^ (static_cast<uint32_t>(static_cast<int32_t>(k) >> 31) ^ 0xffffffffu |
                              0x80000000u));
}

}  // namespace bkv
