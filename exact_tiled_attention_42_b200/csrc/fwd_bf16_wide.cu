// Forward pass for wide heads (d = 192 and 256) on sm_100a, bf16 in, fp32
// accumulate.
//
// The method is the one of fwd_bf16.cu ("FlashAttention: The Algorithm That
// Made Long-Context AI Possible", section "What tiling changes": tiles on
// chip, a running row maximum and sum; "FlashAttention-3: Fast and Accurate
// Attention with Asynchrony and Low-precision", abstract: warp
// specialisation, the softmax of one tile overlapping the matrix products of
// another). What changes is the tiling, because tensor memory holds 512
// columns: two 128-row query tiles would need 2 x 128 score columns plus
// 2 x d output columns, more than 512 once d > 128. So a CTA owns ONE
// 128-row query tile and walks the keys 64 at a time with two score buffers:
//   warp 4      TMA producer: Q once, then K_j and V_j (64 keys x d) through
//               a ring of shared-memory stages with full/empty mbarriers.
//   warp 5      one thread issues every tcgen05 MMA, in the order
//               S_0, S_1, PV_0, S_2, PV_1, S_3, ... : S_{j+2} goes into the
//               buffer PV_j has just read P_j from (MMAs of one thread run in
//               issue order), so the tensor cores compute the next scores
//               while the softmax works on the current ones.
//   warps 0-3   softmax: thread r owns query row r (tensor-memory lane r).
// Per 64-key tile the products cost 2 x 128 x 64 x d x 2 flops against
// 128 x 64 exponentials, so at d >= 192 the tensor cores, not MUFU, bound the
// kernel. Scores are kept in base 2, the running maximum is only raised when
// it grows by more than TAU (the stale maximum enters l and O alike, so the
// result is exact), and a rescale of O waits for the previous P V product to
// have finished writing O.
//
// Tensor memory: S_a [0,64), S_b [64,128) (P, bf16, over the first 32
// columns of its buffer), O [128, 128+d).
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 64;   // keys per tile
constexpr int PRODUCER_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr int THREADS = 192;
constexpr float TAU = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

template <int D>
struct WideCfg {
  static constexpr int BOXES = D / 64;
  static constexpr int QBOX = BM * 128;          // 64 columns x 128 rows, bf16
  static constexpr int KBOX = BN * 128;          // 64 columns x 64 rows
  static constexpr int Q_BYTES = BOXES * QBOX;
  static constexpr int KV_BYTES = BOXES * KBOX;
  static constexpr int NS = (D == 192) ? 3 : 2;  // K and V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * KV_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 2 + 2 + 4;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t COL_S = 0;   // S_a at 0, S_b at 64
  static constexpr uint32_t COL_O = 128;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(COL_O + D <= TMEM_COLS, "tensor memory budget");
};

template <int NS>
struct WBars {
  uint32_t base;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + NS + s); }
  __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * NS + s); }
  __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * NS + s); }
  __device__ uint32_t s_full(int b) const { return base + 8u * (1 + 4 * NS + b); }
  __device__ uint32_t p_full(int b) const { return base + 8u * (3 + 4 * NS + b); }
  __device__ uint32_t pv_done() const { return base + 8u * (5 + 4 * NS); }
  __device__ uint32_t o_final() const { return base + 8u * (6 + 4 * NS); }
  __device__ uint32_t epi() const { return base + 8u * (7 + 4 * NS); }
  __device__ uint32_t teardown() const { return base + 8u * (8 + 4 * NS); }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) break;  // 100 ms
  }
}

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(THREADS, 1)
    fwd_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  using C = WideCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid: heads fastest, the query tiles with the most key tiles (causal)
  // first, so the light tiles form the tail.
  // heads in groups (raster_pairs, one query tile per CTA), heaviest tiles first
  const int BH = static_cast<int>(gridDim.x) / p.num_qtiles;
  int bh, qt;
  raster_pairs(static_cast<int>(blockIdx.x), BH, p.num_qtiles, p.raster_heads, bh, qt);
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  int s0 = 0, n = p.N;
  if (VARLEN) {
    s0 = p.cu_seqlens[b];
    n = p.cu_seqlens[b + 1] - s0;
    if (n < 0 || n > p.N || s0 < 0 || s0 + n > p.total) {
      if (threadIdx.x == 0 && qt == 0) report_status(p.status, FA_ERR_INVALID_ARG | (SITE_SEQLENS << 8));
      return;
    }
    if (qt * BM >= n) return;  // past this sequence's end
  }
  const int qhead = VARLEN ? hq : bh;
  const int kvh = VARLEN ? hq / p.group : b * p.Hkv + hq / p.group;
  const int kv_end = CAUSAL ? min((qt + 1) * BM, n) : n;  // keys [0, kv_end) can be visible
  const int nkv = (kv_end + BN - 1) / BN;
  auto tma_rows = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int x, int r, int head) {
    if (VARLEN)
      tma_load_3d(dst, m, bar, x, head, s0 + r);
    else
      tma_load_3d(dst, m, bar, x, r, head);
  };

  const WBars<C::NS> bars{base + C::OFF_BAR};
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
      mbar_init(bars.p_full(x), 4);  // one arrive per softmax warp
    }
    mbar_init(bars.pv_done(), 1);
    mbar_init(bars.o_final(), 1);
    mbar_init(bars.epi(), 4);
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

  if (warp == PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bars.q_full(), C::Q_BYTES);
      for (int bx = 0; bx < C::BOXES; ++bx)
        tma_rows(base + C::OFF_Q + bx * C::QBOX, &tmQ, bars.q_full(), bx * 64, qt * BM, qhead);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait_sleep(bars.k_empty(s), ph ^ 1, abort, p.status, SITE_K_EMPTY)) break;
        mbar_arrive_expect_tx(bars.k_full(s), C::KV_BYTES);
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_rows(base + C::OFF_K + s * C::KV_BYTES + bx * C::KBOX, &tmK, bars.k_full(s), bx * 64, j * BN, kvh);
        if (!mbar_wait_sleep(bars.v_empty(s), ph ^ 1, abort, p.status, SITE_V_EMPTY)) {
          issued = 2 * j + 1;
          break;
        }
        mbar_arrive_expect_tx(bars.v_full(s), C::KV_BYTES);
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_rows(base + C::OFF_V + s * C::KV_BYTES + bx * C::KBOX, &tmV, bars.v_full(s), bx * 64, j * BN, kvh);
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
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
      const uint32_t sQ = base + C::OFF_Q;
      // S_j = Q K_j^T into buffer j & 1
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::NS;
        if (!mbar_wait_sleep(bars.k_full(s), (j / C::NS) & 1, abort, p.status, SITE_K_FULL)) return false;
        tc_fence_after();
        const uint64_t da = smem_desc_sw128(sQ, 16, 1024);
        const uint64_t db = smem_desc_sw128(base + C::OFF_K + s * C::KV_BYTES, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + C::COL_S + (j & 1) * 64, desc_plus(da, (kk >> 2) * C::QBOX + (kk & 3) * 32),
                 desc_plus(db, (kk >> 2) * C::KBOX + (kk & 3) * 32), IDESC_QK, kk > 0 ? 1u : 0u);
        mma_commit(bars.s_full(j & 1));
        mma_commit(bars.k_empty(s));
        return true;
      };
      bool ok = mbar_wait_sleep(bars.q_full(), 0, abort, p.status, SITE_Q_FULL);
      if (ok) ok = issue_s(0);
      if (ok && nkv > 1) ok = issue_s(1);
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % C::NS;
        if (!mbar_wait_sleep(bars.v_full(s), (j / C::NS) & 1, abort, p.status, SITE_V_FULL)) break;
        if (!mbar_wait_sleep(bars.p_full(j & 1), (j >> 1) & 1, abort, p.status, SITE_P_FULL)) break;
        tc_fence_after();
        const uint64_t dv = smem_desc_sw128(base + C::OFF_V + s * C::KV_BYTES, C::KBOX, 1024);
        // O += P_j V_j: 16 keys per instruction (P: 8 columns of bf16 pairs;
        // V: two 8-row groups of the MN-major 64-row tile)
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + C::COL_O, tmem + C::COL_S + (j & 1) * 64 + kk * 8, desc_plus(dv, kk * 16 * 128), IDESC_PV,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bars.v_empty(s));
        mma_commit(bars.pv_done());
        if (j + 2 < nkv && !issue_s(j + 2)) break;
      }
      mma_commit(bars.o_final());
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-3)
    const int row = warp * 32 + lane;
    const int qrow = qt * BM + row;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::COL_O;
    const float cl2 = p.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = nkv > 0;
    for (int j = 0; ok && j < nkv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bars.s_full(j & 1), (j >> 1) & 1, abort, p.status, SITE_S_FULL))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + C::COL_S + (j & 1) * 64;
      float s[BN];
      {
        uint32_t r[2][32];
        tmem_ld_x32(tS, r[0]);
        tmem_ld_x32(tS + 32, r[1]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(r[c][i]);
      }
      const int kv0 = j * BN;
      if (kv0 + BN > n || (CAUSAL && kv0 + BN - 1 > qt * BM)) {
        const int lim = CAUSAL ? min(qrow + 1, n) : n;  // keys [0, lim) are visible
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= lim) s[c] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = s[i];
#pragma unroll
      for (int c = 8; c < BN; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      const float tile_max = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * cl2;
      if (j == 0) {
        m = tile_max;
      } else if (__any_sync(0xffffffffu, tile_max > m + TAU)) {
        const float m_new = fmaxf(m, tile_max);
        const float alpha = ex2(m - m_new);
        l *= alpha;
        m = m_new;
        // O may still be receiving P_{j-1} V_{j-1}: wait for that product
        if (!__all_sync(0xffffffffu, mbar_wait_sleep(bars.pv_done(), (j - 1) & 1, abort, p.status, SITE_O_DONE))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D; c += 16) {
          uint32_t r[16];
          tmem_ld_x16(tO + c, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st_x16(tO + c, r);
        }
      }
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int qd = 0; qd < 2; ++qd) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = ex2(fmaf(s[qd * 32 + 2 * i], cl2, neg_m));
          const float bb = ex2(fmaf(s[qd * 32 + 2 * i + 1], cl2, neg_m));
          ls[i & 3] += a + bb;
          pk[i] = pack_bf16x2(a, bb);
        }
        tmem_st_x16(tS + qd * 16, pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(j & 1));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.o_final(), 0, abort, p.status, SITE_O_DONE));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const uint32_t stage = base + C::OFF_Q;  // Q is no longer read once every product has finished
      const bool direct = VARLEN && (qt + 1) * BM > n;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld_x32(tO + c, r);
        tmem_wait_ld();
        const uint32_t box = stage + (c >> 6) * C::QBOX;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(r[q * 8 + 2 * e]) * inv_l, __uint_as_float(r[q * 8 + 2 * e + 1]) * inv_l);
          if (direct) {
            if (qrow < n && in_bounds((static_cast<long long>(s0 + qrow) * p.Hq + hq) * D + c + q * 8 + 7,
                                      static_cast<long long>(p.total) * p.Hq * D, p.status, 6))
              *reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(s0 + qrow) * p.Hq + hq) * D + c + q * 8) =
                  make_uint4(w[0], w[1], w[2], w[3]);
          } else {
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + sw128_offset(row, ((c & 63) >> 3) + q)),
                         "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                         : "memory");
          }
        }
      }
      if (!direct) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.epi());
        if (row == 0 && mbar_wait_sleep(bars.epi(), 0, abort, p.status, SITE_O_DONE)) {
          for (int bx = 0; bx < C::BOXES; ++bx) {
            if (VARLEN)
              tma_store_3d(&tmO, stage + bx * C::QBOX, bx * 64, hq, s0 + qt * BM);
            else
              tma_store_3d(&tmO, stage + bx * C::QBOX, bx * 64, qt * BM, bh);
          }
          bulk_commit();
          bulk_wait_read0();
        }
      }
      if (qrow < n) {
        if (VARLEN) {
          const long long li = static_cast<long long>(hq) * p.total + s0 + qrow;
          if (in_bounds(li, static_cast<long long>(p.Hq) * p.total, p.status, 7)) p.lse[li] = (m + __log2f(l)) * LN2;
        } else {
          const long long li = static_cast<long long>(bh) * p.N + qrow;
          if (in_bounds(li, static_cast<long long>(BH) * p.N, p.status, 7)) p.lse[li] = (m + __log2f(l)) * LN2;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
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

template <int D, bool CAUSAL, bool VARLEN>
cudaError_t launch(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmO,
                   const FwdParams& p, int BH, cudaStream_t stream) {
  using C = WideCfg<D>;
  auto kern = fwd_wide_kernel<D, CAUSAL, VARLEN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(BH * p.num_qtiles);
  kern<<<grid, THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmO, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmO,
                     const FwdParams& p, int BH, bool causal, cudaStream_t stream) {
  if (p.cu_seqlens)
    return causal ? launch<D, true, true>(tmQ, tmK, tmV, tmO, p, BH, stream)
                  : launch<D, false, true>(tmQ, tmK, tmV, tmO, p, BH, stream);
  return causal ? launch<D, true, false>(tmQ, tmK, tmV, tmO, p, BH, stream)
                : launch<D, false, false>(tmQ, tmK, tmV, tmO, p, BH, stream);
}

}  // namespace

cudaError_t launch_fwd_wide(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmO, const FwdParams& p, int BH, int d, bool causal,
                            cudaStream_t stream) {
  if (d == 192) return launch_d<192>(tmQ, tmK, tmV, tmO, p, BH, causal, stream);
  return launch_d<256>(tmQ, tmK, tmV, tmO, p, BH, causal, stream);
}

}  // namespace fa
