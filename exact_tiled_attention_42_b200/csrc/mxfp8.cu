// MXFP8 forward of exact softmax attention on sm_100a, d = 128: e4m3
// operands with one power-of-two (E8M0) scale per 32 elements along each
// product's contraction, applied by the tensor cores themselves
// (tcgen05.mma kind::mxf8f6f4 with block scales).
//
// "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
// Low-precision" (abstract) names block quantisation for FP8 without fixing
// the block; this is the reading in which the blocks are the ones B200 scales
// in hardware, per the OCP Microscaling Formats (MX) specification v1.0
// (MXFP8, E4M3 elements, E8M0 shared exponents over 32 elements):
//   Q, K  rows quantised in blocks of 32 columns (contraction of Q K^T),
//         optionally after the rotation diag(sigma) H_d of the FP8 path;
//   V     columns quantised in blocks of 32 keys (contraction of P V);
//   P     each row quantised in blocks of 32 keys, tile by tile, in the
//         softmax warps.
// Shared exponent e = floor(log2 amax) - 8, clamped to [-127, 127] (a zero
// block takes -127); rule "fit" takes one more when amax's significand
// exceeds 1.75, so no element is clamped; rule "ocp" keeps the
// specification's value and saturates at 448.
//
// Forward kernel: the FP8 forward's layout (two 128-row query tiles per CTA,
// a TMA producer warp, one MMA-issuing thread, two softmax warpgroups) on
// 96-key tiles, three MX blocks each: tensor memory then holds both query
// tiles' scores (96 columns, P over the first 24) and outputs (128) with 32
// columns left for each tile's block-scale cells. The next tile's Q K^T is
// issued in two parts: keys 32-95 as soon as the softmax has read S (s_free),
// keys 0-31 (the columns P uses) after P V. A row raises its running max only
// past TAU (log2 units; see TAU).
// Block scales sit in tensor memory as the tensor cores read them: the scale
// of A's row i (and block b along K) in lane i, column base + i/32, byte b;
// the scale of B's column n in lane n % 32 of EVERY lane quarter (the tensor
// cores read it from the quarter of the output row), column base + n/32.
// Each softmax warpgroup writes its own tile's cells (Q once; K of tile j+1
// before it signals s_free; V and P of tile j before p_full), so no cell is
// shared by the two query tiles.
//
// Tensor memory: S0 [0,96), S1 [96,192), O0 [192,320), O1 [320,448); scale
// cells of query tile x from 448 + 32x: Q (4 columns), K (two slots of 4),
// K for keys 32-95 (two slots of 4), V (two slots of 4), P (4).
#include "common.cuh"
#include "kernels.h"
#include "rotation.cuh"

namespace fa {
namespace {

constexpr int D = 128;
constexpr int BM = 128;
constexpr int BN = 96;  // key tile: three 32-key MX blocks
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
// Three warpgroups: softmax of query tile 0 (warps 0-3) and 1 (warps 4-7);
// warpgroup 2 holds the producer and MMA warps. After setup warpgroup 2 lowers
// its registers so the softmax warps can rise (256 * 208 + 128 * 88 =
// 384 * 168, checked against the compiled count before launching).
constexpr int THREADS = 384;
constexpr int REGS_SOFTMAX = 208;
constexpr int REGS_OTHER = 88;
static_assert(256 * REGS_SOFTMAX + 128 * REGS_OTHER <= THREADS * 168, "register split");
// A row raises its running max only past TAU (log2 units). MX block scales
// absorb any magnitude of P, so TAU bounds accuracy, not range: a stale max
// leaves the row's largest term off the exact code 2^8 (P = 1) and, under the
// specification's rule, open to the clamp at 448. Measured on the emulation
// (N = 1000-2048, 0.1 % outliers, 96-key tiles): RMS error against exact
// attention within 0.6 % (TAU = 2) / 3.4 % (TAU = 4) / 11 % (TAU = 8) of the
// one-tile schedule; TAU = 4 rescales O in about a fifth of the key tiles of
// a 4096-key row (TAU = 8: a twentieth, TAU = 0: four fifths).
constexpr float TAU = 4.0f;
constexpr float LN2 = 0.69314718055994530942f;

// ------------------------------------------------------------------ helpers
// MX shared exponent of a block whose largest magnitude is amax.
__device__ __forceinline__ int mx_exponent(float amax, int fit) {
  const uint32_t bits = __float_as_uint(amax);
  const int E = static_cast<int>((bits >> 23) & 0xFFu);
  if (!(amax > 0.f) || E == 0) return -127;  // zero or subnormal: below the E8M0 range after the -8
  int e = E - 127 - 8;
  if (fit && (bits & 0x7FFFFFu) > 0x600000u) e += 1;  // significand above 1.75
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}
// 2^-e as a float, for e in [-127, 126].
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float(static_cast<uint32_t>(127 - e) << 23); }

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(lo) : "f"(b), "f"(a));
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// ------------------------------------------------------------------ pre-pass
// One CTA per 64-row block of one (batch, head) of Q, K or V (grid z): 8 warps
// x 8 rows, d/32 = 4 consecutive elements per lane. Q, K: the 8 lanes holding
// one 32-column block share its exponent (shuffles). V: a block is 32 keys of
// one column: per-warp column maxima meet in shared memory; V's exponents are
// stored one 4-byte word per 96-key tile and column (the forward's tiles).
__global__ void __launch_bounds__(256) mxfp8_quant_kernel(const MxParams p) {
  constexpr int E = D / 32;
  const int t = blockIdx.z;  // 0 = Q, 1 = K, 2 = V
  const int bh = blockIdx.y;
  const int blk = blockIdx.x;
  if (bh >= p.heads[t]) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool rot = p.rotate && t < 2;
  __shared__ float colmax[8][D];

  float sig[E];
  if (rot) rotation_signs<E>(sig, p.rotation_seed, lane);

  float y[8][E];
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
      for (int e = 0; e < E; ++e) y[rr][e] = __double2float_rn(x[e]);
    }
  }
  if (t < 2) {
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int n = blk * 64 + warp * 8 + rr;
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(y[rr][e]));
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (n >= p.N) continue;
      const int ex = mx_exponent(amax, p.fit);
      const float inv = pow2_neg(ex);
      const long long r = static_cast<long long>(bh) * p.N + n;
      if (!in_bounds(r, static_cast<long long>(p.heads[t]) * p.N, p.status, 13)) continue;
      *reinterpret_cast<uint32_t*>(p.codes[t] + r * D + lane * E) =
          e4m3x4(__fmul_rn(y[rr][0], inv), __fmul_rn(y[rr][1], inv), __fmul_rn(y[rr][2], inv), __fmul_rn(y[rr][3], inv));
      if ((lane & 7) == 0) p.exps[t][r * 4 + (lane >> 3)] = static_cast<uint8_t>(ex + 127);
    }
  } else {
    // V: block = 32 keys (warps 0-3 or 4-7) x one column
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float m = 0.f;
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) m = fmaxf(m, fabsf(y[rr][e]));
      colmax[warp][lane * E + e] = m;
    }
    __syncthreads();
    const int w0 = (warp >> 2) * 4;  // first warp of this warp's 32-key block
    const int kb = blk * 2 + (warp >> 2);  // key block index
    float inv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane * E + e;
      const float amax = fmaxf(fmaxf(colmax[w0][c], colmax[w0 + 1][c]), fmaxf(colmax[w0 + 2][c], colmax[w0 + 3][c]));
      const int ex = mx_exponent(amax, p.fit);
      inv[e] = pow2_neg(ex);
      // one 4-byte word per 96-key tile and column: bytes 0-2 the tile's three
      // 32-key blocks, byte 3 zero
      if ((warp & 3) == 0 && kb < 3 * p.num_ktiles &&
          in_bounds((static_cast<long long>(bh) * D + c) * p.vexp_stride + (kb / 3) * 4 + 3,
                    static_cast<long long>(p.heads[2]) * D * p.vexp_stride, p.status, 14)) {
        uint8_t* w = p.exps[2] + (static_cast<long long>(bh) * D + c) * p.vexp_stride + (kb / 3) * 4;
        w[kb % 3] = static_cast<uint8_t>(ex + 127);
        if (kb % 3 == 2) w[3] = 0;
      }
    }
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int n = blk * 64 + warp * 8 + rr;
      if (n >= p.N || !in_bounds(static_cast<long long>(bh) * p.N + n, static_cast<long long>(p.heads[2]) * p.N, p.status, 15))
        continue;
      *reinterpret_cast<uint32_t*>(p.codes[2] + (static_cast<long long>(bh) * p.N + n) * D + lane * E) =
          e4m3x4(__fmul_rn(y[rr][0], inv[0]), __fmul_rn(y[rr][1], inv[1]), __fmul_rn(y[rr][2], inv[2]),
                 __fmul_rn(y[rr][3], inv[3]));
    }
  }
}

// ------------------------------------------------------------------ forward
struct Cfg {
  static constexpr int Q_BYTES = BM * D;   // e4m3: 128 rows x 128 bytes
  static constexpr int KV_BYTES = BN * D;  // 96 rows x 128 bytes
  static constexpr int NS = 3;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_O = OFF_V + NS * KV_BYTES;  // bf16 output staging, 2 x 32 KB
  static constexpr int O_TILE_BYTES = BM * D * 2;
  static constexpr int OFF_BAR = OFF_O + 2 * O_TILE_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 14;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  // Tensor memory: scores of query tiles 0/1 (96 columns each, P over the
  // first 24), outputs (128 each), then the block-scale cells of each query
  // tile: Q (4 columns), K (two slots of 4: keys 0-31, 32-63, 64-95), K for
  // the split-off keys 32-95 (two slots of 4: a scale address must sit on a
  // 4-column boundary, so that part cannot start one column into K's slot),
  // V (two slots of 4), P (4).
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 96, COL_O0 = 192, COL_O1 = 320;
  static constexpr uint32_t COL_SF = 448, SF_PER_TILE = 32;
  static constexpr uint32_t SF_Q = 0, SF_K = 4, SF_KT = 12, SF_V = 20, SF_P = 28;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(COL_SF + 2 * SF_PER_TILE <= TMEM_COLS, "tensor memory budget");
  static_assert(OFF_K % 1024 == 0 && KV_BYTES % 1024 == 0 && OFF_O % 1024 == 0, "128B-swizzle atoms");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Bars {
  uint32_t base;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + Cfg::NS + s); }
  __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * Cfg::NS + s); }
  __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * Cfg::NS + s); }
  __device__ uint32_t s_full(int x) const { return base + 8u * (1 + 4 * Cfg::NS + x); }
  __device__ uint32_t p_full(int x) const { return base + 8u * (3 + 4 * Cfg::NS + x); }
  __device__ uint32_t o_done(int x) const { return base + 8u * (5 + 4 * Cfg::NS + x); }
  __device__ uint32_t epi(int x) const { return base + 8u * (7 + 4 * Cfg::NS + x); }
  // the softmax of query tile x has read S_x: the columns past P's may take the next S_x
  __device__ uint32_t s_free(int x) const { return base + 8u * (9 + 4 * Cfg::NS + x); }
  // query tile x's first scale cells (Q, K of tiles 0) are written
  __device__ uint32_t sf_ready(int x) const { return base + 8u * (11 + 4 * Cfg::NS + x); }
  __device__ uint32_t teardown() const { return base + 8u * (13 + 4 * Cfg::NS); }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) break;  // 100 ms
  }
}

// Instruction descriptor of kind::mxf8f6f4 with E8M0 block scales: e4m3 A and
// B (format 0), fp32 D; bits [4,6) B's scale byte, 15/16 A/B major, [17,23)
// N >> 3, 23 scale type (1 = E8M0), [24,29) M >> 4, [29,31) A's scale byte.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, bool b_mn_major, int sf_id) {
  return (static_cast<uint32_t>(sf_id) << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (1u << 23) | (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

__device__ __forceinline__ void mma_mx_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_mx_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], [%1], %2, %3, [%4], [%5], p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_st_x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

template <bool CAUSAL>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_mxfp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const MxParams p) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // heads in groups (raster_pairs), the pairs of query tiles with the most
  // key tiles first
  const int BH = static_cast<int>(gridDim.x) / p.num_pairs;
  int bh, pair;
  raster_pairs(static_cast<int>(blockIdx.x), BH, p.num_pairs, p.raster_heads, bh, pair);
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  const int kvh = b * p.Hkv + hq / p.group;
  const int qt0 = 2 * pair, qt1 = 2 * pair + 1;
  const bool has1 = qt1 < p.num_qtiles;
  auto ntiles = [&](int qt) { return ((CAUSAL ? min((qt + 1) * BM, p.N) : p.N) + BN - 1) / BN; };
  const int n0 = ntiles(qt0);
  const int n1 = has1 ? ntiles(qt1) : 0;
  const int nkv = n0 > n1 ? n0 : n1;

  const Bars bars{base + C::OFF_BAR};
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + C::NUM_BARS * 8);
  volatile int* const abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full(), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bars.k_full(s), 1);
      mbar_init(bars.k_empty(s), 1);
      mbar_init(bars.v_full(s), 1);
      mbar_init(bars.v_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bars.s_full(x), 1);
      mbar_init(bars.p_full(x), 4);
      mbar_init(bars.o_done(x), 1);
      mbar_init(bars.epi(x), 4);
      mbar_init(bars.s_free(x), 4);
      mbar_init(bars.sf_ready(x), 4);
    }
    mbar_init(bars.teardown(), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    setmaxnreg_dec<REGS_OTHER>();
    if (warp == PRODUCER_WARP) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bars.q_full(), (has1 ? 2 : 1) * C::Q_BYTES);
        tma_load_3d(base + C::OFF_Q, &tmQ, bars.q_full(), 0, qt0 * BM, bh);
        if (has1) tma_load_3d(base + C::OFF_Q + C::Q_BYTES, &tmQ, bars.q_full(), 0, qt1 * BM, bh);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % C::NS;
          const uint32_t ph = (j / C::NS) & 1;
          if (!mbar_wait_sleep(bars.k_empty(s), ph ^ 1, abort, p.status, SITE_K_EMPTY)) break;
          mbar_arrive_expect_tx(bars.k_full(s), C::KV_BYTES);
          tma_load_3d(base + C::OFF_K + s * C::KV_BYTES, &tmK, bars.k_full(s), 0, j * BN, kvh);
          if (!mbar_wait_sleep(bars.v_empty(s), ph ^ 1, abort, p.status, SITE_V_EMPTY)) {
            issued = 2 * j + 1;
            break;
          }
          mbar_arrive_expect_tx(bars.v_full(s), C::KV_BYTES);
          tma_load_3d(base + C::OFF_V + s * C::KV_BYTES, &tmV, bars.v_full(s), 0, j * BN, kvh);
          issued = 2 * j + 2;
        }
        if (*abort) {
          drain_wait(bars.q_full(), 0);
          for (int t = (issued > 2 * C::NS ? issued - 2 * C::NS : 0); t < issued; ++t) {
            const int j = t >> 1;
            drain_wait((t & 1) ? bars.v_full(j % C::NS) : bars.k_full(j % C::NS), (j / C::NS) & 1);
          }
        }
      }
    } else if (warp == MMA_WARP) {
      if (lane == 0) {
        const uint32_t sQ = base + C::OFF_Q;
        // S_x(j) over keys [key0, key0 + N) of the stage into their score
        // columns; K's scale cells of tile j in slot j & 1 (keys 0-95, or the
        // copy for keys 32-95)
        auto issue_qk = [&](int x, int j, int key0, int N_) {
          const int stage = j % C::NS;
          const uint32_t sf = tmem + C::COL_SF + x * C::SF_PER_TILE;
          const uint64_t da = smem_desc_sw128(sQ + x * C::Q_BYTES, 16, 1024);
          const uint64_t db = smem_desc_sw128(base + C::OFF_K + stage * C::KV_BYTES + key0 * 128, 16, 1024);
          const uint32_t sfb = sf + (key0 == 32 ? C::SF_KT : C::SF_K) + (j & 1) * 4;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_mx_ss(tmem + (x ? C::COL_S1 : C::COL_S0) + key0, desc_plus(da, kk * 32), desc_plus(db, kk * 32),
                      N_ == 32 ? idesc_mx(BM, 32, false, kk) : (N_ == 64 ? idesc_mx(BM, 64, false, kk) : idesc_mx(BM, BN, false, kk)),
                      sf + C::SF_Q, sfb, kk > 0 ? 1u : 0u);
        };
        // O_x += P_x(j) V(j): 32 keys per instruction (P: 8 columns of four
        // e4m3; V: four 8-row groups of the MN-major tile), key block kk's scale byte
        auto issue_pv = [&](int x, int j, bool accumulate) {
          const int stage = j % C::NS;
          const uint32_t sf = tmem + C::COL_SF + x * C::SF_PER_TILE;
          const uint64_t dv = smem_desc_sw128(base + C::OFF_V + stage * C::KV_BYTES, 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)
            mma_mx_ts(tmem + (x ? C::COL_O1 : C::COL_O0), tmem + (x ? C::COL_S1 : C::COL_S0) + kk * 8,
                      desc_plus(dv, kk * 4096), idesc_mx(BM, D, true, kk), sf + C::SF_P, sf + C::SF_V + (j & 1) * 4,
                      (accumulate || kk > 0) ? 1u : 0u);
        };
        bool ok = mbar_wait_sleep(bars.q_full(), 0, abort, p.status, SITE_Q_FULL) &&
                  mbar_wait_sleep(bars.k_full(0), 0, abort, p.status, SITE_K_FULL) &&
                  mbar_wait_sleep(bars.sf_ready(0), 0, abort, p.status, SITE_P_FULL) &&
                  (n1 == 0 || mbar_wait_sleep(bars.sf_ready(1), 0, abort, p.status, SITE_P_FULL));
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0, 0, BN);
          mma_commit(bars.s_full(0));
          if (n1 > 0) {
            issue_qk(1, 0, 0, BN);
            mma_commit(bars.s_full(1));
          }
          mma_commit(bars.k_empty(0));
        }
        for (int j = 1; ok && j <= nkv; ++j) {
          const int vs = (j - 1) % C::NS;
          const int ks = j % C::NS;
          if (!mbar_wait_sleep(bars.v_full(vs), ((j - 1) / C::NS) & 1, abort, p.status, SITE_V_FULL)) break;
          if (j < nkv && !mbar_wait_sleep(bars.k_full(ks), (j / C::NS) & 1, abort, p.status, SITE_K_FULL)) break;
          tc_fence_after();
          // S_x(j) for keys 32-95 (columns P does not use) once the softmax has
          // read S_x(j-1) and written K's scales of tile j
          for (int x = 0; ok && x < 2; ++x) {
            if (j >= (x ? n1 : n0)) continue;
            if (!mbar_wait_sleep(bars.s_free(x), (j - 1) & 1, abort, p.status, SITE_P_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(x, j, 32, BN - 32);
          }
          for (int x = 0; ok && x < 2; ++x) {
            const int nx = x ? n1 : n0;
            if (j - 1 >= nx) continue;
            if (!mbar_wait_sleep(bars.p_full(x), (j - 1) & 1, abort, p.status, SITE_P_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(x, j - 1, j > 1);
            if (j < nx) {
              issue_qk(x, j, 0, 32);  // keys 0-31, over P's columns, after P V has read P
              mma_commit(bars.s_full(x));
            } else {
              mma_commit(bars.o_done(x));
            }
          }
          if (!ok) break;
          if (j < nkv) mma_commit(bars.k_empty(ks));
          mma_commit(bars.v_empty(vs));
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (warpgroups 0 and 1)
    setmaxnreg_inc<REGS_SOFTMAX>();
    const int x = warp >> 2;
    const int qt = x ? qt1 : qt0;
    const int n = x ? n1 : n0;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qrow = qt * BM + row;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + (x ? C::COL_S1 : C::COL_S0);
    const uint32_t tO = tmem + lane_off + (x ? C::COL_O1 : C::COL_O0);
    const uint32_t tSF = tmem + lane_off + C::COL_SF + x * C::SF_PER_TILE;
    const float cl2 = p.score_log2;
    const uint32_t* kexp = reinterpret_cast<const uint32_t*>(p.exps[1]) + static_cast<long long>(kvh) * p.N;
    const uint32_t* vexp = reinterpret_cast<const uint32_t*>(p.exps[2]) + static_cast<long long>(kvh) * D * (p.vexp_stride / 4);
    // K's scale cells of tile j (slot j & 1): key n of the tile in lane n % 32
    // of every lane quarter, column n / 32, and the same for keys 32-95 alone
    // (the split-off part of the next S); this warp writes its quarter
    auto write_k_scales = [&](int j) {
      uint32_t c[3];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int key = j * BN + 32 * q + lane;
        c[q] = key < p.N && in_bounds(static_cast<long long>(kvh) * p.N + key, static_cast<long long>(p.heads[1]) * p.N,
                                      p.status, 16)
                   ? kexp[key]
                   : 0u;
      }
      tmem_st_x4(tSF + C::SF_K + (j & 1) * 4, c[0], c[1], c[2], 0u);
      tmem_st_x4(tSF + C::SF_KT + (j & 1) * 4, c[1], c[2], 0u, 0u);
    };
    // V's scale cells of tile j (slot j & 1): column d in lane d % 32 of every
    // quarter, column d / 32; bytes 0-2 the tile's three key blocks
    auto write_v_scales = [&](int j) {
      uint32_t c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[q] = in_bounds((static_cast<long long>(kvh) * D + 32 * q + lane) * (p.vexp_stride / 4) + j,
                         static_cast<long long>(p.heads[2]) * D * (p.vexp_stride / 4), p.status, 17)
                   ? vexp[(32 * q + lane) * (p.vexp_stride / 4) + j]
                   : 0u;
      tmem_st_x4(tSF + C::SF_V + (j & 1) * 4, c[0], c[1], c[2], c[3]);
    };
    if (n > 0) {
      // Q's scale cell: row i in lane i, column i / 32
      tmem_st_x1(tSF + C::SF_Q + wq,
                 qrow < p.N && in_bounds(static_cast<long long>(bh) * p.N + qrow, static_cast<long long>(p.heads[0]) * p.N,
                                         p.status, 18)
                     ? reinterpret_cast<const uint32_t*>(p.exps[0])[static_cast<long long>(bh) * p.N + qrow]
                     : 0u);
      write_k_scales(0);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.sf_ready(x));
    }

    float m = -INFINITY;  // running max of c s, as m + mlo (mlo: m's rounding residual)
    float mlo = 0.f;
    float l = 0.f;
    bool ok = n > 0;
    for (int j = 0; ok && j < n; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bars.s_full(x), j & 1, abort, p.status, SITE_S_FULL))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
      {
        uint32_t r[3][32];
#pragma unroll
        for (int c = 0; c < 3; ++c) tmem_ld_x32(tS + 32 * c, r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[c][i]);
      }
      // S is in registers and tile j+1's K scales go into the slot S_x(j-1)
      // used: the MMA warp may start the next S_x
      if (j + 1 < n) {
        write_k_scales(j + 1);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_free(x));
      const int kv0 = j * BN;
      if (kv0 + BN > p.N || (CAUSAL && kv0 + BN - 1 > qt * BM)) {
        const int lim = CAUSAL ? min(qrow + 1, p.N) : p.N;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= lim) s[c] = -INFINITY;
      }
      const float smax = row_max<BN>(s);
      const float tile_max = smax * cl2;
      const float tile_lo = tile_max > -INFINITY ? fmaf(smax, cl2, -tile_max) : 0.f;  // exact: c smax = tile_max + tile_lo
      if (j == 0) {
        m = tile_max;
        mlo = tile_lo;
      } else {
        const bool raise = tile_max > m + TAU;
        if (__any_sync(0xffffffffu, raise)) {
          // O_x is stable: S_x(j) completed after P_x(j-1) V(j-1)
          const float m_new = raise ? tile_max : m;
          const float mlo_new = raise ? tile_lo : mlo;
          const float alpha = ex2((m - m_new) + (mlo - mlo_new));
          l *= alpha;
          m = m_new;
          mlo = mlo_new;
#pragma unroll
          for (int c = 0; c < D; c += 16) {
            uint32_t r[16];
            tmem_ld_x16(tO + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st_x16(tO + c, r);
          }
        }
      }
      // P = 2^(c s - m) in fp32, x = fl(fma(s, c, -m) - mlo) (exactly 0 at the
      // key that set the max); its MX blocks of 32 keys: exponent from the
      // block's largest P, codes e4m3(P 2^-e)
      const float nm = (m == -INFINITY) ? 0.f : -m;
      const float2 c2 = make_float2(cl2, cl2), nm2 = make_float2(nm, nm), nlo2 = make_float2(-mlo, -mlo);
      float2 lsum = make_float2(0.f, 0.f);
      uint32_t pk[24];
      uint32_t pexp = 0;
#pragma unroll
      for (int blk = 0; blk < 3; ++blk) {
        float pv[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 xx = __fadd2_rn(__ffma2_rn(make_float2(s[32 * blk + 2 * i], s[32 * blk + 2 * i + 1]), c2, nm2), nlo2);
          pv[2 * i] = ex2(xx.x);
          pv[2 * i + 1] = ex2(xx.y);
          lsum = __fadd2_rn(lsum, make_float2(pv[2 * i], pv[2 * i + 1]));
        }
        const int ex = mx_exponent(row_max<32>(pv), p.fit);
        const float inv = pow2_neg(ex);  // a power of two: P 2^-e is exact
        const float2 inv2 = make_float2(inv, inv);
        pexp |= static_cast<uint32_t>(ex + 127) << (8 * blk);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 a = __fmul2_rn(make_float2(pv[4 * i], pv[4 * i + 1]), inv2);
          const float2 c = __fmul2_rn(make_float2(pv[4 * i + 2], pv[4 * i + 3]), inv2);
          pk[8 * blk + i] = e4m3x4(a.x, a.y, c.x, c.y);
        }
      }
      l += lsum.x + lsum.y;
      tmem_st_x16(tS, *reinterpret_cast<const uint32_t(*)[16]>(pk));
      tmem_st_x8(tS + 16, pk + 16);
      tmem_st_x1(tSF + C::SF_P + wq, pexp);
      write_v_scales(j);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(x));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bars.o_done(x), 0, abort, p.status, SITE_O_DONE));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const uint32_t stage = base + C::OFF_O + x * C::O_TILE_BYTES;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld_x32(tO + c, r);
        tmem_wait_ld();
        const uint32_t box = stage + (c >> 6) * (BM * 128);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w4[e] = pack_bf16x2(__uint_as_float(r[q * 8 + 2 * e]) * inv_l, __uint_as_float(r[q * 8 + 2 * e + 1]) * inv_l);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + sw128_offset(row, ((c & 63) >> 3) + q)),
                       "r"(w4[0]), "r"(w4[1]), "r"(w4[2]), "r"(w4[3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.epi(x));
      if (row == 0 && mbar_wait(bars.epi(x), 0, abort, p.status, SITE_O_DONE)) {
        tma_store_3d(&tmO, stage, 0, qt * BM, bh);
        tma_store_3d(&tmO, stage + BM * 128, 64, qt * BM, bh);
        bulk_commit();
        bulk_wait_read0();
      }
      if (qrow < p.N && in_bounds(static_cast<long long>(bh) * p.N + qrow, static_cast<long long>(p.heads[0]) * p.N,
                                  p.status, 19))
        p.lse[static_cast<size_t>(bh) * p.N + qrow] = ((m + mlo) + __log2f(l)) * LN2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    if (*abort) {
      if (lane == 0) {
        mma_commit(bars.teardown());
        drain_wait(bars.teardown(), 0);
      }
      __syncwarp();
    }
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <bool CAUSAL>
cudaError_t launch_fwd(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmO,
                       const MxParams& p, int BH, cudaStream_t stream) {
  auto kern = fwd_mxfp8_kernel<CAUSAL>;
  // The softmax warpgroups' setmaxnreg.inc waits until the CTA's register
  // pool has room; make sure the compiled launch allocation covers the split.
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes attr;
    cudaError_t ea = cudaFuncGetAttributes(&attr, kern);
    if (ea != cudaSuccess) return ea;
    regs = attr.numRegs;
  }
  if (256 * REGS_SOFTMAX + 128 * REGS_OTHER > THREADS * regs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<dim3(BH * p.num_pairs), THREADS, Cfg::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmO, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mxfp8_quant(const MxParams& p, cudaStream_t stream) {
  const int maxh = p.heads[0] > p.heads[1] ? p.heads[0] : p.heads[1];
  dim3 grid((3 * p.num_ktiles + 1) / 2, maxh, 3);  // 64-row blocks covering every 96-key tile
  mxfp8_quant_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fwd_mxfp8(const CUtensorMap& tmQ8, const CUtensorMap& tmK8, const CUtensorMap& tmV8,
                             const CUtensorMap& tmO, const MxParams& p, int BH, bool causal, cudaStream_t stream) {
  return causal ? launch_fwd<true>(tmQ8, tmK8, tmV8, tmO, p, BH, stream)
                : launch_fwd<false>(tmQ8, tmK8, tmV8, tmO, p, BH, stream);
}

}  // namespace fa
