// Incoherent processing shared by the FP8 and MXFP8 pre-passes: the rotation
// y = x diag(sigma) H_d of one row, H_d the Sylvester Hadamard matrix and
// sigma a +-1 vector from SplitMix64 (Steele, Lea and Flood 2014) of the seed
// ("FlashAttention-3: Fast and Accurate Attention with Asynchrony and
// Low-precision", abstract, names the rotation without its form).
// sigma_t = +1 when the top bit of output t of the seed's stream 5 is clear;
// the same sigma for Q and K, so (Q R)(K R)^T = d Q K^T and the 1/d goes into
// the softmax scale. The row is spread over a warp, E = D / 32 consecutive
// elements per lane, in fp64 (every sum of bf16 inputs is exact there): a
// fast Walsh-Hadamard transform with in-lane butterflies, then shuffles.
#pragma once

#include <cstdint>

namespace fa {

constexpr uint64_t SM_GAMMA = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t splitmix_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
// Output number `i` (0-based) of SplitMix64 seeded with `seed`.
__device__ __forceinline__ uint64_t splitmix_at(uint64_t seed, uint64_t i) {
  return splitmix_mix(seed + (i + 1) * SM_GAMMA);
}

// sigma for this lane's E consecutive columns.
template <int E>
__device__ __forceinline__ void rotation_signs(float (&sig)[E], uint64_t rotation_seed, int lane) {
  const uint64_t key = splitmix_at(rotation_seed, 5);
#pragma unroll
  for (int e = 0; e < E; ++e) sig[e] = (splitmix_at(key, lane * E + e) >> 63) ? -1.f : 1.f;
}

// x <- x diag(sigma) H_D for the row whose columns lane * E .. lane * E + E - 1
// this lane holds (all 32 lanes of the warp take part).
template <int E, int D>
__device__ __forceinline__ void hadamard_row(double (&x)[E], const float (&sig)[E], int lane) {
#pragma unroll
  for (int e = 0; e < E; ++e) x[e] *= sig[e];
  // in-lane butterflies (h < E), then across lanes (h >= E)
#pragma unroll
  for (int h = 1; h < E; h <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (!(e & h)) {
        const double a = x[e], b = x[e + h];
        x[e] = a + b;
        x[e + h] = a - b;
      }
#pragma unroll
  for (int h = E; h < D; h <<= 1) {
    const int lm = h / E;
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const double other = __shfl_xor_sync(0xffffffffu, x[e], lm);
      x[e] = upper ? other - x[e] : x[e] + other;
    }
  }
}

}  // namespace fa
