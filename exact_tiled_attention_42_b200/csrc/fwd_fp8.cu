// FP8 (e4m3) forward of exact softmax attention on sm_100a, d = 128.
//
// Same CTA layout as the bf16 forward (two 128-row query tiles, TMA producer
// warp, one MMA-issuing thread, two softmax warpgroups), on the operands the
// FP8 pre-pass wrote: e4m3 Q and K (rotated) and V, each with one fp32 scale
// per 64-row block. "FlashAttention-3: Fast and Accurate Attention with
// Asynchrony and Low-precision" (abstract) describes FP8 with block
// quantisation; the forms used here:
//   S = sQ(row block) sK(key block) (Qc Kc^T) scale / d       (kind::f8f6f4)
//   running max and sum as in the bf16 path, but a row raises its max once a
//   tile's max exceeds it by more than TAU = 0.8 (not 8), so P <= 2^0.8;
//   P~ = e4m3(P * sV(key block) / max sV * 256)               (V's block scale
//        folded into P so that one MMA sums over key blocks with different
//        scales; the 256 keeps small probabilities above e4m3's subnormals)
//   O = (sum P~ Vc) * max sV / 256 / l,   l = sum of unquantised P.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512); P~ (4 e4m3 per
// column) over the first 32 columns of its S. The next S_x is issued in two
// parts: the keys over columns 32-127 as soon as the softmax has read S_x into
// registers (s_free), overlapping that softmax; the keys over P's columns
// after P V has read P.
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int BM = 128;
constexpr int BN = 128;
// P overwrites the first P_COLS score columns of its tile (e4m3, four keys per
// 32-bit column), so only the keys of those columns wait for P V to have read P.
constexpr int P_COLS = BN / 4;
constexpr int D = 128;
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
// Three full warpgroups: softmax of query tile 0 (warps 0-3) and tile 1
// (warps 4-7); warpgroup 2 holds the producer and MMA warps and two warps
// with no role. After setup warpgroup 2 lowers its registers (setmaxnreg)
// so the softmax warps can hold their score row without spilling past the
// 168 a thread is launched with: 256 * 208 + 128 * 88 = 384 * 168, checked
// against the compiled register count on the host before launching.
constexpr int THREADS = 384;
constexpr int REGS_SOFTMAX = 208;
constexpr int REGS_OTHER = 88;
static_assert(256 * REGS_SOFTMAX + 128 * REGS_OTHER <= THREADS * 168, "register split");
constexpr float LN2 = 0.69314718055994530942f;
constexpr float P_LIFT = 256.f;
// A row raises its running max only when a tile's max exceeds it by more than
// TAU (log2 units): P then stays below 2^TAU and P w below 2^TAU * 256 =
// 445.7, inside e4m3's range.
constexpr float TAU = 0.8f;
static_assert(P_LIFT * 1.7411011f <= 448.f, "2^TAU * P_LIFT must stay within e4m3's range");
// Of every 8 groups of 4 scores, this many take their exponentials on the FMA
// pipe (exp2_poly) instead of MUFU: the two query tiles' 2 x 128 x 128
// exponentials per key tile need 2048 MUFU cycles against about 1080 of e4m3
// MMA, but the polynomial costs issue slots the softmax also needs. Measured
// on the FP8 workload (forward alone, next S split around P's columns):
// 0 -> 1223, 1 -> 1223, 2 -> 1195, 3 -> 1113 TFLOP/s.
constexpr int POLY_GROUPS = 1;

// exp2_poly on two values with packed FMA-pipe arithmetic.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  return make_float2(exp2_poly(x.x), exp2_poly(x.y));
}

struct Cfg {
  static constexpr int TILE_BYTES = BM * D;  // e4m3: 128 rows x 128 bytes
  static constexpr int NS = 3;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NS * TILE_BYTES;
  static constexpr int OFF_O = OFF_V + NS * TILE_BYTES;  // bf16 output staging, 2 x 32 KB
  static constexpr int O_TILE_BYTES = BM * D * 2;
  static constexpr int OFF_BAR = OFF_O + 2 * O_TILE_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 11;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 384;
  static constexpr uint32_t TMEM_COLS = 512;
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
  __device__ uint32_t teardown() const { return base + 8u * (7 + 4 * Cfg::NS); }
  __device__ uint32_t epi(int x) const { return base + 8u * (8 + 4 * Cfg::NS + x); }
  // the softmax of query tile x has read S_x into registers: the score
  // columns past P's may take the next tile's S
  __device__ uint32_t s_free(int x) const { return base + 8u * (10 + 4 * Cfg::NS + x); }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) break;  // 100 ms
  }
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(lo) : "f"(b), "f"(a));
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <bool CAUSAL>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const Fp8Params p) {
  using C = Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid in groups of heads (raster_pairs): inside a group the pairs with
  // the most key tiles (causal) come first, heads fastest.
  const int BH = static_cast<int>(gridDim.x) / p.num_pairs;
  int bh, pair;
  raster_pairs(static_cast<int>(blockIdx.x), BH, p.num_pairs, p.raster_heads, bh, pair);
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  const int kvh = b * p.Hkv + hq / p.group;
  const int qt0 = 2 * pair, qt1 = 2 * pair + 1;
  const bool has1 = qt1 < p.num_qtiles;
  const int n0 = CAUSAL ? qt0 + 1 : p.num_qtiles;
  const int n1 = has1 ? (CAUSAL ? qt1 + 1 : p.num_qtiles) : 0;
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
    // warpgroup 2: producer, MMA issuer and two warps without a role
    setmaxnreg_dec<REGS_OTHER>();
    if (warp == PRODUCER_WARP) {
      if (lane == 0) {
        const uint32_t sQ = base + C::OFF_Q;
        mbar_arrive_expect_tx(bars.q_full(), (has1 ? 2 : 1) * C::TILE_BYTES);
        tma_load_3d(sQ, &tmQ, bars.q_full(), 0, qt0 * BM, bh);
        if (has1) tma_load_3d(sQ + C::TILE_BYTES, &tmQ, bars.q_full(), 0, qt1 * BM, bh);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % C::NS;
          const uint32_t ph = (j / C::NS) & 1;
          if (!mbar_wait_sleep(bars.k_empty(s), ph ^ 1, abort, p.status, SITE_K_EMPTY)) break;
          mbar_arrive_expect_tx(bars.k_full(s), C::TILE_BYTES);
          tma_load_3d(base + C::OFF_K + s * C::TILE_BYTES, &tmK, bars.k_full(s), 0, j * BN, kvh);
          if (!mbar_wait_sleep(bars.v_empty(s), ph ^ 1, abort, p.status, SITE_V_EMPTY)) {
            issued = 2 * j + 1;
            break;
          }
          mbar_arrive_expect_tx(bars.v_full(s), C::TILE_BYTES);
          tma_load_3d(base + C::OFF_V + s * C::TILE_BYTES, &tmV, bars.v_full(s), 0, j * BN, kvh);
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
        constexpr uint32_t IDESC_QK = idesc_e4m3(BM, BN, false, false);
        constexpr uint32_t IDESC_QK_HEAD = idesc_e4m3(BM, P_COLS, false, false);
        constexpr uint32_t IDESC_QK_TAIL = idesc_e4m3(BM, BN - P_COLS, false, false);
        constexpr uint32_t IDESC_PV = idesc_e4m3(BM, D, false, true);
        const uint32_t sQ = base + C::OFF_Q;
        // S_x = Q_x K^T over keys [key0, key0 + N) of the stage, into the
        // score columns of those keys (128-byte K rows: key0 * 128 bytes is a
        // whole number of 8-row swizzle atoms)
        auto issue_qk = [&](int x, int stage, int key0, uint32_t idesc) {
          const uint32_t dS = tmem + (x ? C::COL_S1 : C::COL_S0) + key0;
          const uint64_t da = smem_desc_sw128(sQ + x * C::TILE_BYTES, 16, 1024);
          const uint64_t db = smem_desc_sw128(base + C::OFF_K + stage * C::TILE_BYTES + key0 * 128, 16, 1024);
  #pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)  // 32 e4m3 = 32 bytes of each 128-byte row
            mma_ss_f8(dS, desc_plus(da, kk * 32), desc_plus(db, kk * 32), idesc, kk > 0 ? 1u : 0u);
        };
        auto issue_pv = [&](int x, int stage, bool accumulate) {
          const uint32_t dO = tmem + (x ? C::COL_O1 : C::COL_O0);
          const uint32_t aP = tmem + (x ? C::COL_S1 : C::COL_S0);
          const uint64_t dv = smem_desc_sw128(base + C::OFF_V + stage * C::TILE_BYTES, 16384, 1024);
  #pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)  // 32 keys = four 8-row groups; 32 e4m3 of P = 8 columns
            mma_ts_f8(dO, aP + kk * 8, desc_plus(dv, kk * 4096), IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
        };
        bool ok = mbar_wait_sleep(bars.q_full(), 0, abort, p.status, SITE_Q_FULL) &&
                  mbar_wait_sleep(bars.k_full(0), 0, abort, p.status, SITE_K_FULL);
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0, 0, IDESC_QK);
          mma_commit(bars.s_full(0));
          if (n1 > 0) {
            issue_qk(1, 0, 0, IDESC_QK);
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
          // S_x(j) for the keys whose score columns P does not use, as soon as
          // the softmax has read S_x(j-1): it overlaps that softmax
          for (int x = 0; ok && x < 2; ++x) {
            if (j >= (x ? n1 : n0)) continue;
            if (!mbar_wait_sleep(bars.s_free(x), (j - 1) & 1, abort, p.status, SITE_P_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(x, ks, P_COLS, IDESC_QK_TAIL);
          }
          for (int x = 0; ok && x < 2; ++x) {
            const int nx = x ? n1 : n0;
            if (j - 1 >= nx) continue;
            if (!mbar_wait_sleep(bars.p_full(x), (j - 1) & 1, abort, p.status, SITE_P_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(x, vs, j > 1);
            if (j < nx) {
              // the keys over P's columns, once P V has read P (in order)
              issue_qk(x, ks, 0, IDESC_QK_HEAD);
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
    // warpgroups 0 and 1: softmax
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
    const float* sQs = p.scales[0] + static_cast<long long>(bh) * p.nblk;
    const float* sKs = p.scales[1] + static_cast<long long>(kvh) * p.nblk;
    const float* sVs = p.scales[2] + static_cast<long long>(kvh) * p.nblk;
    // the head's largest V block scale (every lane computes it; L1-served)
    float vmax = 0.f;
    for (int i = lane; i < p.nblk; i += 32)
      if (in_bounds(static_cast<long long>(kvh) * p.nblk + i, static_cast<long long>(p.heads[2]) * p.nblk, p.status, 8))
        vmax = fmaxf(vmax, sVs[i]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    const float wlift = P_LIFT / vmax;
    const float crow = p.score_log2 * sQs[min(qrow, p.N - 1) >> 6];
    float m = -INFINITY;  // running max of the log2-domain scores, as m + mlo (mlo: m's rounding residual)
    float mlo = 0.f;
    float l = 0.f;
    bool ok = n > 0;
    for (int j = 0; ok && j < n; ++j) {
      // this tile's block scales, loaded while S is still being computed
      const int kb0 = 2 * j;  // key blocks of this tile: 2j (keys 0-63) and 2j+1 (64-127)
      const int kb1 = min(2 * j + 1, p.nblk - 1);
      const bool kb_ok = in_bounds(static_cast<long long>(kvh) * p.nblk + kb1, static_cast<long long>(p.heads[1]) * p.nblk,
                                   p.status, 9);
      const float sk0 = kb_ok ? sKs[kb0] : 1.f, sk1 = kb_ok ? sKs[kb1] : 1.f;
      const float sv0 = kb_ok ? sVs[kb0] : 1.f, sv1 = kb_ok ? sVs[kb1] : 1.f;
      if (!__all_sync(0xffffffffu, mbar_wait(bars.s_full(x), j & 1, abort, p.status, SITE_S_FULL))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BN];
      {
        // all four loads in flight before the single wait
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_x32(tS + 32 * c, r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[c][i]);
      }
      // S is in registers: the MMA warp may write the next S over the columns
      // P will not use
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.s_free(x));
      // log2-domain score factor of each key half (folded into the FFMA
      // before the exponential); the max is taken on raw scores per half
      const float f0 = crow * sk0, f1 = crow * sk1;
      const float w0 = sv0 * wlift, w1 = sv1 * wlift;
      const int kv0 = j * BN;
      const bool edge = (kv0 + BN > p.N) || (CAUSAL && kv0 + BN - 1 > qt * BM);
      if (edge) {
        const int lim = CAUSAL ? min(qrow + 1, p.N) : p.N;
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= lim) s[c] = -INFINITY;
      }
      // row maxima of the two key halves (three-input max)
      const float smax0 = row_max<64>(s);
      const float smax1 = row_max<64>(s + 64);
      const float t0 = smax0 * f0, t1 = smax1 * f1;
      const bool top1 = t1 > t0;
      const float tile_max = top1 ? t1 : t0;
      // exact residual of the largest product: f smax = tile_max + tile_lo
      const float tile_lo = tile_max > -INFINITY ? (top1 ? fmaf(smax1, f1, -t1) : fmaf(smax0, f0, -t0)) : 0.f;
      if (j == 0) {
        m = tile_max;
        mlo = tile_lo;
      } else {
        // a row raises its max only past TAU; the warp rescales O in tensor
        // memory when any of its rows did (alpha = 1 for the others)
        const bool raise = tile_max > m + TAU;
        if (__any_sync(0xffffffffu, raise)) {
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
      // P~ = 2^(c s - m), two scores per packed FMA; then P~ w with one
      // packed multiply. (Folding log2 w into the exponent would save the
      // multiply, but P~ = 1 for a row's largest key, and 2^(log2 w) is not
      // exactly w: where w sits on an e4m3 rounding tie -- block scales are
      // ratios of short bf16 values, so it can -- the code would flip.)
      // x = fl(fma(s, f, -m) - mlo): the fused product-minus-max is exact at
      // the key that set the max (it equals mlo there), so that key gets
      // x = 0 and P = 1 exactly whatever the compiler fuses (otherwise the
      // product's rounding residual survives and P w can round off an e4m3
      // tie the other way)
      const float nm = (m == -INFINITY) ? 0.f : -m;
      const float2 f0v = make_float2(f0, f0), f1v = make_float2(f1, f1), nmv = make_float2(nm, nm);
      const float2 nlov = make_float2(-mlo, -mlo);
      const float2 w0v = make_float2(w0, w0), w1v = make_float2(w1, w1);
      float2 lsum[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const bool hi = i >= 16;
        const float2 x01 = __fadd2_rn(__ffma2_rn(make_float2(s[4 * i], s[4 * i + 1]), hi ? f1v : f0v, nmv), nlov);
        const float2 x23 = __fadd2_rn(__ffma2_rn(make_float2(s[4 * i + 2], s[4 * i + 3]), hi ? f1v : f0v, nmv), nlov);
        float2 a01, a23;
        if ((i & 7) < POLY_GROUPS) {
          a01 = exp2_poly2(x01);
          a23 = exp2_poly2(x23);
        } else {
          a01 = make_float2(ex2(x01.x), ex2(x01.y));
          a23 = make_float2(ex2(x23.x), ex2(x23.y));
        }
        lsum[i & 1] = __fadd2_rn(lsum[i & 1], __fadd2_rn(a01, a23));
        const float2 q01 = __fmul2_rn(a01, hi ? w1v : w0v), q23 = __fmul2_rn(a23, hi ? w1v : w0v);
        pk[i] = e4m3x4(q01.x, q01.y, q23.x, q23.y);
      }
      tmem_st_x32(tS, pk);
      l += (lsum[0].x + lsum[0].y) + (lsum[1].x + lsum[1].y);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(x));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bars.o_done(x), 0, abort, p.status, SITE_O_DONE));
    if (ok) {
      tc_fence_after();
      const float out_mul = vmax / P_LIFT / l;
      const uint32_t stage = base + C::OFF_O + x * C::O_TILE_BYTES;
#pragma unroll
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
            w4[e] = pack_bf16x2(__uint_as_float(r[q * 8 + 2 * e]) * out_mul,
                                __uint_as_float(r[q * 8 + 2 * e + 1]) * out_mul);
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
                                  p.status, 10))
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
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmO,
                   const Fp8Params& p, int BH, cudaStream_t stream) {
  auto kern = fwd_fp8_kernel<CAUSAL>;
  // The softmax warpgroups' setmaxnreg.inc waits until the CTA's register
  // pool has room; make sure the compiled launch allocation covers the split.
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa_attr;
    cudaError_t e0 = cudaFuncGetAttributes(&fa_attr, kern);
    if (e0 != cudaSuccess) return e0;
    regs = fa_attr.numRegs;
  }
  if (256 * REGS_SOFTMAX + 128 * REGS_OTHER > THREADS * regs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(BH * p.num_pairs);
  kern<<<grid, THREADS, Cfg::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmO, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_fp8(const CUtensorMap& tmQ8, const CUtensorMap& tmK8, const CUtensorMap& tmV8,
                           const CUtensorMap& tmO, const Fp8Params& p, int BH, bool causal, cudaStream_t stream) {
  return causal ? launch<true>(tmQ8, tmK8, tmV8, tmO, p, BH, stream)
                : launch<false>(tmQ8, tmK8, tmV8, tmO, p, BH, stream);
}

}  // namespace fa
