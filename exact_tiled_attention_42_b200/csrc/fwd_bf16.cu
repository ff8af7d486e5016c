// Forward pass of exact softmax attention on sm_100a (bf16 in, fp32 accumulate).
//
// Method: "FlashAttention: The Algorithm That Made Long-Context AI Possible"
// (promptingindex.com), section "What tiling changes": Q, K and V are cut into
// tiles that live on chip, each key tile updates a running row maximum and a
// running sum of exponentials, and only O (plus the row log-sum-exp) is
// written. "FlashAttention-2: Faster Attention with Better Parallelism and
// Work Partitioning" (abstract) adds the work split used here: thread blocks
// over query tiles even for one head, rows of a tile owned by distinct threads
// so no partial outputs are reduced across warps, and fewer non-matmul
// operations. "FlashAttention-3: Fast and Accurate Attention with Asynchrony
// and Low-precision" (abstract) describes overlapping data movement with the
// tensor cores by warp specialisation and interleaving the softmax of one tile
// with the matrix products of another; the B200 form of both is below.
//
// One CTA owns two 128-row query tiles of one (batch, head) and walks the key
// tiles of that head:
//   warp 8      TMA producer: Q tiles once, then K_j and V_j through a ring of
//               shared-memory stages guarded by full/empty mbarriers.
//   warp 9      one thread issues every tcgen05 MMA: S_x = Q_x K_j^T (both
//               operands in shared memory, fp32 result in tensor memory) and
//               O_x += P_x V_j (P_x read from tensor memory).
//   warps 0-3   softmax of query tile 0, warps 4-7 of query tile 1: thread r
//               owns row r of its tile (tensor-memory lane r).
// While one tile's softmax runs on the CUDA cores, the tensor cores run the
// other tile's products (ping-pong). Scores are kept in base 2
// (c = scale * log2 e, one FFMA per score before ex2). The running maximum is
// only raised when a tile's maximum exceeds it by more than TAU (log2 units);
// P then stays below 2^TAU, the same stale maximum enters both l and O so the
// result is exact, and the rescale of O in tensor memory is skipped on most
// tiles. O is divided by l once, in the epilogue. P (bf16) overwrites the
// first half of its own S columns in tensor memory.
//
// Tensor memory (512 columns x 128 lanes, fp32): S0 [0,128), S1 [128,256),
// O0 [256, 256+d), O1 [256+d, 256+2d).
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int BM = 128;  // query rows per tile (tcgen05 M)
constexpr int BN = 128;  // keys per tile
constexpr int PRODUCER_WARP = 8;
constexpr int MMA_WARP = 9;
// Three full warpgroups: softmax of query tile 0 (warps 0-3) and tile 1
// (warps 4-7); warpgroup 2 holds the producer and MMA warps and two warps
// with no role. After setup warpgroup 2 gives registers back (setmaxnreg)
// so the softmax warps, which keep a 128-score row each, can grow past the
// 168 a thread is launched with (three warps share each scheduler's
// register file) without spilling. The split adds up to the launch
// allocation exactly: 256 * 208 + 128 * 88 = 384 * 168; the host checks the
// compiled register count against it before launching.
constexpr int FWD_THREADS = 384;
constexpr int REGS_SOFTMAX = 208;
constexpr int REGS_OTHER = 88;
constexpr int REGS_AT_LAUNCH = 168;
static_assert(256 * REGS_SOFTMAX + 128 * REGS_OTHER <= FWD_THREADS * REGS_AT_LAUNCH, "register split");
constexpr float TAU = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

template <int D>
struct FwdCfg {
  static constexpr int BOX_BYTES = BM * 128;        // one 64-column x 128-row bf16 box
  static constexpr int BOXES = D / 64;
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr int NS = (D == 64) ? 3 : 2;      // K and V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NS * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NS * TILE_BYTES;
  static constexpr int NUM_BARS = 1 + 4 * NS + 9;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Bars {
  uint32_t base;
  int ns;
  __device__ uint32_t q_full() const { return base; }
  __device__ uint32_t k_full(int s) const { return base + 8u * (1 + s); }
  __device__ uint32_t k_empty(int s) const { return base + 8u * (1 + ns + s); }
  __device__ uint32_t v_full(int s) const { return base + 8u * (1 + 2 * ns + s); }
  __device__ uint32_t v_empty(int s) const { return base + 8u * (1 + 3 * ns + s); }
  __device__ uint32_t s_full(int x) const { return base + 8u * (1 + 4 * ns + x); }
  __device__ uint32_t p_full(int x) const { return base + 8u * (3 + 4 * ns + x); }
  __device__ uint32_t o_done(int x) const { return base + 8u * (5 + 4 * ns + x); }
  __device__ uint32_t teardown() const { return base + 8u * (7 + 4 * ns); }
  __device__ uint32_t epi(int x) const { return base + 8u * (8 + 4 * ns + x); }
};

// Wait bounded by time only (ignores the abort flag): used on the way out to
// let in-flight copies and MMAs land before shared or tensor memory is freed.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) break;  // 100 ms
  }
}

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(FWD_THREADS, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid in groups of heads (raster_pairs): inside a group the pairs with
  // the most key tiles (causal) come first, heads fastest.
  const int BH = static_cast<int>(gridDim.x) / p.num_pairs;
  int bh, pair;  // bh = b * Hq + hq
  raster_pairs(static_cast<int>(blockIdx.x), BH, p.num_pairs, p.raster_heads, bh, pair);
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  // A packed batch's sequence b: tokens s0 .. s0 + len - 1 (its own N). CTAs
  // whose query tiles lie past the sequence's end leave at once.
  int s0 = 0, len = p.N;
  if (VARLEN) {
    s0 = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - s0;
    if (len < 0 || len > p.N || s0 < 0 || s0 + len > p.total) {
      if (threadIdx.x == 0 && pair == 0) report_status(p.status, FA_ERR_INVALID_ARG | (SITE_SEQLENS << 8));
      return;
    }
  }
  const int num_qtiles = VARLEN ? (len + BM - 1) / BM : p.num_qtiles;
  const int qt0 = 2 * pair;
  const int qt1 = 2 * pair + 1;
  if (VARLEN && qt0 >= num_qtiles) return;
  // head coordinates of the TMA maps: [B*H, N, d] (fixed) or [T, H, d] (packed)
  const int qhead = VARLEN ? hq : bh;
  const int kvh = VARLEN ? hq / p.group : b * p.Hkv + hq / p.group;
  const bool has1 = qt1 < num_qtiles;
  const int n0 = CAUSAL ? qt0 + 1 : num_qtiles;
  const int n1 = has1 ? (CAUSAL ? qt1 + 1 : num_qtiles) : 0;
  const int nkv = n0 > n1 ? n0 : n1;
  // TMA coordinates of 128 rows starting at row r of a head (fixed: y = row,
  // z = head; packed: y = head, z = token)
  auto tma_rows = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int x, int r, int head) {
    if (VARLEN)
      tma_load_3d(dst, m, bar, x, head, s0 + r);
    else
      tma_load_3d(dst, m, bar, x, r, head);
  };

  const Bars bars{base + C::OFF_BAR, C::NS};
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
      mbar_init(bars.o_done(x), 1);
      mbar_init(bars.epi(x), 4);  // one arrive per softmax warp once its O rows are staged
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
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        const uint32_t sQ = base + C::OFF_Q;
        mbar_arrive_expect_tx(bars.q_full(), (has1 ? 2 : 1) * C::TILE_BYTES);
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_rows(sQ + bx * C::BOX_BYTES, &tmQ, bars.q_full(), bx * 64, qt0 * BM, qhead);
        if (has1)
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_rows(sQ + C::TILE_BYTES + bx * C::BOX_BYTES, &tmQ, bars.q_full(), bx * 64, qt1 * BM, qhead);
        int issued = 0;
        for (int j = 0; j < nkv; ++j) {
          const int s = j % C::NS;
          const uint32_t ph = (j / C::NS) & 1;
          if (!mbar_wait_sleep(bars.k_empty(s), ph ^ 1, abort, p.status, SITE_K_EMPTY)) break;
          mbar_arrive_expect_tx(bars.k_full(s), C::TILE_BYTES);
          const uint32_t sK = base + C::OFF_K + s * C::TILE_BYTES;
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_rows(sK + bx * C::BOX_BYTES, &tmK, bars.k_full(s), bx * 64, j * BN, kvh);
          if (!mbar_wait_sleep(bars.v_empty(s), ph ^ 1, abort, p.status, SITE_V_EMPTY)) {
            issued = 2 * j + 1;
            break;
          }
#ifdef FA_DEBUG_WITHHOLD
          // Debug build only: leave the first V tile out, so that the MMA
          // warp's bounded wait for it runs out (the test of the abort path).
          if (p.debug_withhold && j == 0) {
            issued = 2 * j + 2;
            continue;
          }
#endif
          mbar_arrive_expect_tx(bars.v_full(s), C::TILE_BYTES);
          const uint32_t sV = base + C::OFF_V + s * C::TILE_BYTES;
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_rows(sV + bx * C::BOX_BYTES, &tmV, bars.v_full(s), bx * 64, j * BN, kvh);
          issued = 2 * j + 2;
        }
        if (*abort) {
          // Let every copy already issued land before the CTA can exit.
          drain_wait(bars.q_full(), 0);
          for (int t = (issued > 2 * C::NS ? issued - 2 * C::NS : 0); t < issued; ++t) {
#ifdef FA_DEBUG_WITHHOLD
            if (p.debug_withhold && t == 1) continue;  // the V tile that was never issued
#endif
            const int j = t >> 1;
            const uint32_t bar = (t & 1) ? bars.v_full(j % C::NS) : bars.k_full(j % C::NS);
            drain_wait(bar, (j / C::NS) & 1);
          }
        }
      }
    } else if (warp == MMA_WARP) {
      // ------------------------------------------------------------ MMA issue
      if (lane == 0) {
        constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false, false);
        constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, false, true);
        const uint32_t sQ = base + C::OFF_Q;
        auto issue_qk = [&](int x, int stage) {
          const uint32_t dS = tmem + (x ? C::COL_S1 : C::COL_S0);
          const uint64_t da = smem_desc_sw128(sQ + x * C::TILE_BYTES, 16, 1024);
          const uint64_t db = smem_desc_sw128(base + C::OFF_K + stage * C::TILE_BYTES, 16, 1024);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
            mma_ss(dS, desc_plus(da, off), desc_plus(db, off), IDESC_QK, kk > 0 ? 1u : 0u);
          }
        };
        auto issue_pv = [&](int x, int stage, bool accumulate) {
          const uint32_t dO = tmem + (x ? C::COL_O1 : C::COL_O0);
          const uint32_t aP = tmem + (x ? C::COL_S1 : C::COL_S0);
          const uint64_t dv = smem_desc_sw128(base + C::OFF_V + stage * C::TILE_BYTES, C::BOX_BYTES, 1024);
  #pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // 16 keys = two 8-row groups of the MN-major V tile; 16 bf16 of P = 8 columns.
            mma_ts(dO, aP + kk * 8, desc_plus(dv, kk * 16 * 128), IDESC_PV, (accumulate || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = mbar_wait_sleep(bars.q_full(), 0, abort, p.status, SITE_Q_FULL) &&
                  mbar_wait_sleep(bars.k_full(0), 0, abort, p.status, SITE_K_FULL);
        if (ok) {
          tc_fence_after();
          issue_qk(0, 0);
          mma_commit(bars.s_full(0));
          if (n1 > 0) {
            issue_qk(1, 0);
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
          for (int x = 0; x < 2; ++x) {
            const int nx = x ? n1 : n0;
            if (j - 1 >= nx) continue;
            if (!mbar_wait_sleep(bars.p_full(x), (j - 1) & 1, abort, p.status, SITE_P_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(x, vs, j > 1);
            if (j < nx) {
              issue_qk(x, ks);
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
    // ------------------------------------------------------------ softmax
    const int x = warp >> 2;  // query tile of this warpgroup
    const int qt = x ? qt1 : qt0;
    const int n = x ? n1 : n0;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int qrow = qt * BM + row;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + (x ? C::COL_S1 : C::COL_S0);
    const uint32_t tO = tmem + lane_off + (x ? C::COL_O1 : C::COL_O0);
    const float cl2 = p.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    bool ok = n > 0;
    for (int j = 0; ok && j < n; ++j) {
      // Every lane polls; the outcome is made warp-uniform before the
      // .sync.aligned tensor-memory instructions that follow.
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bars.s_full(x), j & 1, abort, p.status, SITE_S_FULL))) {
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
      const int kv0 = j * BN;
      const bool edge = (kv0 + BN > len) || (CAUSAL && kv0 + BN - 1 > qt * BM);
      if (edge) {
        const int lim = CAUSAL ? min(qrow + 1, len) : len;  // keys [0, lim) are visible
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kv0 + c >= lim) s[c] = -INFINITY;
      }
      const float tile_max = row_max<BN>(s) * cl2;
      if (j == 0) {
        m = tile_max;
      } else if (__any_sync(0xffffffffu, tile_max > m + TAU)) {
        const float m_new = fmaxf(m, tile_max);
        const float alpha = ex2(m - m_new);
        l *= alpha;
        m = m_new;
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
      // P = 2^(c s - m), two scores per packed FMA and add
      const float neg_m = (m == -INFINITY) ? 0.f : -m;
      const float2 c2 = make_float2(cl2, cl2), nm2 = make_float2(neg_m, neg_m);
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 xx = __ffma2_rn(make_float2(s[qd * 32 + 2 * i], s[qd * 32 + 2 * i + 1]), c2, nm2);
          const float2 ab = make_float2(ex2(xx.x), ex2(xx.y));
          ls[i & 1] = __fadd2_rn(ls[i & 1], ab);
          pk[i] = pack_bf16x2(ab.x, ab.y);
        }
        tmem_st_x16(tS + qd * 16, pk);
      }
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_full(x));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.o_done(x), 0, abort, p.status, SITE_O_DONE));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const uint32_t stage = base + C::OFF_Q + x * C::TILE_BYTES;  // Q_x is no longer read
      // A packed batch's last, partial query tile is written row by row: a
      // tile-wide store would reach into the next sequence's rows.
      const bool direct = VARLEN && (qt + 1) * BM > len;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld_x32(tO + c, r);
        tmem_wait_ld();
        const uint32_t box = stage + (c >> 6) * C::BOX_BYTES;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(r[q * 8 + 2 * e]) * inv_l, __uint_as_float(r[q * 8 + 2 * e + 1]) * inv_l);
          if (direct) {
            if (qrow < len && c + q * 8 < p.d &&
                in_bounds((static_cast<long long>(s0 + qrow) * p.Hq + hq) * p.d + c + q * 8 + 7,
                          static_cast<long long>(p.total) * p.Hq * p.d, p.status, 4))
              *reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(s0 + qrow) * p.Hq + hq) * p.d + c + q * 8) =
                  make_uint4(w[0], w[1], w[2], w[3]);
          } else {
            const uint32_t chunk = ((c & 63) >> 3) + q;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + sw128_offset(row, chunk)), "r"(w[0]),
                         "r"(w[1]), "r"(w[2]), "r"(w[3])
                         : "memory");
          }
        }
      }
      if (!direct) {
        // Staged rows -> async proxy, then one thread stores the tile with
        // TMA (rows at or past N and columns past d are clipped by the map).
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.epi(x));
        if (row == 0 && mbar_wait_sleep(bars.epi(x), 0, abort, p.status, SITE_O_DONE)) {
          for (int bx = 0; bx < C::BOXES; ++bx) {
            if (VARLEN)
              tma_store_3d(&tmO, stage + bx * C::BOX_BYTES, bx * 64, hq, s0 + qt * BM);
            else
              tma_store_3d(&tmO, stage + bx * C::BOX_BYTES, bx * 64, qt * BM, bh);
          }
          bulk_commit();
          bulk_wait_read0();
        }
      }
      if (qrow < len) {
        if (VARLEN) {
          const long long li = static_cast<long long>(hq) * p.total + s0 + qrow;
          if (in_bounds(li, static_cast<long long>(p.Hq) * p.total, p.status, 5)) p.lse[li] = (m + __log2f(l)) * LN2;
        } else {
          const long long li = static_cast<long long>(bh) * p.N + qrow;
          if (in_bounds(li, static_cast<long long>(BH) * p.N, p.status, 5)) p.lse[li] = (m + __log2f(l)) * LN2;
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
  using C = FwdCfg<D>;
  auto kern = fwd_bf16_kernel<D, CAUSAL, VARLEN>;
  // The softmax warpgroups' setmaxnreg.inc waits until the CTA's register
  // pool has room; make sure the compiled launch allocation covers the split.
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa_attr;
    cudaError_t e0 = cudaFuncGetAttributes(&fa_attr, kern);
    if (e0 != cudaSuccess) return e0;
    regs = fa_attr.numRegs;
  }
  if (256 * REGS_SOFTMAX + 128 * REGS_OTHER > FWD_THREADS * regs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(BH * p.num_pairs);
  kern<<<grid, FWD_THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmO, p);
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

cudaError_t launch_fwd_bf16(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmO, const FwdParams& p, int BH, int d, bool causal,
                            cudaStream_t stream) {
  if (d == 64) return launch_d<64>(tmQ, tmK, tmV, tmO, p, BH, causal, stream);
  return launch_d<128>(tmQ, tmK, tmV, tmO, p, BH, causal, stream);  // d = 96 or 128
}

}  // namespace fa
