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
//   pair      hash32(seed, b, h, i, u) = mix(k_i ^ (u * G)), u = j >> 1
// One mix decides the two adjacent keys 2u and 2u+1 of row i: element (i, j)
// of head (b, h) is kept iff its 16-bit half -- the low half of the pair's
// hash for even j, the high half for odd j -- is >= T, T = ceil(p * 2^16)
// computed on the host in double precision (0 <= T <= 2^16); survivors are
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

// the hash of key pair u = j >> 1 of a row
__host__ __device__ __forceinline__ uint32_t dropout_hash(uint32_t row_key, uint32_t u) {
  return mix32(row_key ^ (u * kGolden));
}

// keep decisions of the pair's even key (low half) and odd key (high half)
__host__ __device__ __forceinline__ bool keep_lo(uint32_t w, uint32_t threshold) { return (w & 0xffffu) >= threshold; }
__host__ __device__ __forceinline__ bool keep_hi(uint32_t w, uint32_t threshold) { return (w >> 16) >= threshold; }

}  // namespace fa
