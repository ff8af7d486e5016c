// FP8 pre-pass: incoherent processing and block quantisation of Q, K and V.
//
// "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
// Low-precision" (abstract) names block quantisation (a scale per block
// instead of per tensor) and incoherent processing (rotating Q and K so that
// outliers spread before quantising) without giving either's form. Here:
//   - rotation y = x diag(sigma) H_d, H_d the Sylvester Hadamard matrix, sigma
//     a +-1 vector from SplitMix64 (Steele, Lea and Flood 2014) of the seed:
//     sigma_t = +1 when the top bit of output t of stream 5 is clear. The same
//     sigma for Q and K, so (Q R)(K R)^T = d Q K^T; the 1/d goes into the
//     softmax scale. V is not rotated.
//   - y is computed with a fast Walsh-Hadamard transform in fp64, where every
//     sum of bf16 inputs is exact, then rounded once to fp32.
//   - one fp32 scale per block of 64 rows x d of one (batch, head):
//     s = amax / 448 (s = 1 for an all-zero block); codes = e4m3(y * (448 /
//     amax)), round to nearest even, saturating. Each step is one correctly
//     rounded fp32 operation, so the codes are a fixed function of the inputs.
// One CTA quantises one 64-row block: 8 warps x 8 rows, one row per warp at a
// time, d/32 consecutive elements per lane. HBM-bound.
#include "common.cuh"
#include "kernels.h"
#include "rotation.cuh"

namespace fa {
namespace {

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(256) fp8_quant_kernel(const Fp8Params p) {
  constexpr int E = D / 32;  // elements per lane
  const int t = blockIdx.z;  // 0 = Q, 1 = K, 2 = V
  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  if (bh >= p.heads[t]) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool rot = p.rotate && t < 2;
  __shared__ float warp_max[8];

  float sig[E];
  if (rot) rotation_signs<E>(sig, p.rotation_seed, lane);

  float y[8][E];
  float amax = 0.f;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int n = blk * 64 + warp * 8 + rr;
#pragma unroll
    for (int e = 0; e < E; ++e) y[rr][e] = 0.f;
    if (n < p.N) {
      const uint16_t* row = p.src[t] + (static_cast<long long>(bh) * p.N + n) * D + lane * E;
      double x[E];
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = static_cast<double>(__uint_as_float(static_cast<uint32_t>(row[e]) << 16));
      if (rot) hadamard_row<E, D>(x, sig, lane);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        y[rr][e] = __double2float_rn(x[e]);
        amax = fmaxf(amax, fabsf(y[rr][e]));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 1.f;
  if (threadIdx.x == 0 && in_bounds(static_cast<long long>(bh) * p.nblk + blk, static_cast<long long>(p.heads[t]) * p.nblk,
                                     p.status, 11))
    p.scales[t][static_cast<long long>(bh) * p.nblk + blk] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int n = blk * 64 + warp * 8 + rr;
    if (n >= p.N) continue;
    if (!in_bounds((static_cast<long long>(bh) * p.N + n) * D + lane * E + E - 1, static_cast<long long>(p.heads[t]) * p.N * D,
                   p.status, 12))
      continue;
    uint8_t* out = p.codes[t] + (static_cast<long long>(bh) * p.N + n) * D + lane * E;
    if (E == 4) {
      const uint32_t lo = e4m3x2(__fmul_rn(y[rr][0], inv), __fmul_rn(y[rr][1], inv));
      const uint32_t hi = e4m3x2(__fmul_rn(y[rr][2], inv), __fmul_rn(y[rr][3], inv));
      *reinterpret_cast<uint32_t*>(out) = lo | (hi << 16);
    } else {
      *reinterpret_cast<uint16_t*>(out) = e4m3x2(__fmul_rn(y[rr][0], inv), __fmul_rn(y[rr][1], inv));
    }
  }
}

}  // namespace

cudaError_t launch_fp8_quant(const Fp8Params& p, cudaStream_t stream) {
  int maxh = p.heads[0] > p.heads[1] ? p.heads[0] : p.heads[1];
  dim3 grid(p.nblk, maxh, 3);
  fp8_quant_kernel<128><<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fa
