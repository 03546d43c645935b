// dropout_hash.cuh -- the counter-based dropout mask, device side.
//
// The pages say only that dropout is fused into the attention kernel
// ("FlashAttention for Efficient Training", section 3, Fused Kernel Design);
// the generator is this library's own definition (all arithmetic mod 2^32):
//   mix(x):  x ^= x >> 16; x *= C1; x ^= x >> 15; x *= C2; x ^= x >> 16
//   C1 = floor(frac(sqrt 2) * 2^32) = 0x6a09e667
//   C2 = floor(frac(sqrt 3) * 2^32) = 0xbb67ae85
//   G  = floor(2^32 / golden ratio) = 0x9e3779b9
//   row key   k_i = mix(mix(mix(mix(mix(lo32(seed) ^ G) ^ hi32(seed)) ^ b) ^ h) ^ i)
//   element   hash32(seed, b, h, i, j) = mix(k_i ^ (j * G))
// Element (i, j) of head (b, h) is kept iff hash32 >= T with
// T = ceil(p * 2^32) computed on the host in double precision; survivors are
// scaled by 1/(1-p).  The mask is applied after the softmax, so the row sums
// and the logsumexp use the undropped probabilities.
#pragma once

#include <stdint.h>

namespace fa {

constexpr uint32_t kMixC1 = 0x6a09e667u;
constexpr uint32_t kMixC2 = 0xbb67ae85u;
constexpr uint32_t kGolden = 0x9e3779b9u;

__host__ __device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= kMixC1;
  x ^= x >> 15;
  x *= kMixC2;
  x ^= x >> 16;
  return x;
}

__host__ __device__ __forceinline__ uint32_t dropout_row_key(uint64_t seed, uint32_t b, uint32_t h,
                                                             uint32_t i) {
  uint32_t k = mix32(static_cast<uint32_t>(seed) ^ kGolden);
  k = mix32(k ^ static_cast<uint32_t>(seed >> 32));
  k = mix32(k ^ b);
  k = mix32(k ^ h);
  return mix32(k ^ i);
}

__host__ __device__ __forceinline__ uint32_t dropout_hash(uint32_t row_key, uint32_t j) {
  return mix32(row_key ^ (j * kGolden));
}

}  // namespace fa
