// Backward pass of exact softmax attention on sm_100a by recomputation.
//
// The pages say that the tiled algorithm trains Transformers faster
// ("FlashAttention: Fast and Memory-Efficient Exact Attention with
// IO-Awareness", abstract) but give no backward pass. The one here is the
// analytic gradient of O = softmax(scale Q K^T) V, with P rebuilt tile by tile
// from Q, K and the forward's log-sum-exp so that no N x N matrix is stored:
//     P  = exp(scale S - LSE)            dV += P^T dO
//     dP = dO V^T                        dS  = P * (dP - D),  D = rowsum(dO * O)
//     dK += scale dS^T Q                 dQ += scale dS K
// Three kernels: a preprocess (D, -LSE log2 e, zero the fp32 dQ accumulator),
// the main kernel, and a postprocess (dQ = scale * accumulator -> bf16).
//
// Main kernel: one CTA per (128-key tile j, KV head). It keeps K_j and V_j in
// shared memory and dK_j, dV_j in tensor memory, and loops over the query
// heads that share the KV head and over the query tiles i (i >= j when
// causal), so dK and dV are summed over the group without atomics. Per step,
// everything is "transposed" so that keys sit on the 128 tensor-memory lanes:
//   S^T  = K_j Q_i^T      (shared x shared -> tensor memory)
//   dP^T = V_j dO_i^T     (shared x shared -> tensor memory)
//   dV  += P^T dO_i       (P^T from tensor memory, bf16)
//   dK  += dS^T Q_i       (dS^T from tensor memory, bf16)
//   dQ_i = dS K_j         (dS from shared memory, MN-major)
// issued in the order dP^T(i), dV(i), S^T(i+1), dK(i), dQ(i): the next S^T
// starts as soon as dV has read P^T, so the compute warps form P^T(i+1) while
// the tensor cores run dK(i) and dQ(i).
// Roles, 512 threads in four warpgroups: warpgroups 0 and 1 turn S^T into P^T
// and dP^T into dS^T (thread = key row; query columns [0,64) and [64,128), so
// two warps per scheduler share the exponentials); warpgroup 2 drains dQ_i out
// of tensor memory and adds it into the fp32 accumulator with TMA reduce-add
// (thread = query row), apart from the compute warps so that its reduce waits
// never hold up the next P^T; in warpgroup 3, warp 12 loads with TMA and one
// thread of warp 13 issues every MMA. A thread is launched with 128 registers
// (four warps share each scheduler's register file); after setup warpgroup 3
// lowers itself to 88 (setmaxnreg), the compute warpgroups rise to 136 and
// the drain to 152 -- 256 * 136 + 128 * 152 + 128 * 88 = 512 * 128, checked
// against the compiled register count on the host before launching.
// Each compute warpgroup writes its P^T (bf16) over the first 32 of its 64
// S^T columns (and keeps it in registers for dS, since the next S^T lands in
// those columns) and its dS^T over the first 32 of its 64 dP^T columns; for
// d = 128 the dQ accumulator then reuses the dP^T columns, and dS reuses the
// shared-memory slot of dO_i once dV has read it. dK is issued as soon as
// dS^T is in tensor memory, before dS has reached shared memory (which waits
// for dV), and dQ once it has.
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int BT = 128;  // keys per CTA tile; queries per step
constexpr int PRODUCER_WARP = 12;
constexpr int MMA_WARP = 13;
constexpr int BWD_THREADS = 512;
constexpr int REGS_COMPUTE = 136;
constexpr int REGS_DRAIN = 152;
constexpr int REGS_OTHER = 88;
static_assert(256 * REGS_COMPUTE + 128 * REGS_DRAIN + 128 * REGS_OTHER <= BWD_THREADS * 128, "register split");
constexpr float LOG2E = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int BOX_BYTES = 128 * 128;  // 64 bf16 columns x 128 rows
  static constexpr int BOXES = D / 64;
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  static constexpr bool DS_ALIAS = (D == 128);
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + TILE_BYTES;    // 2 slots
  static constexpr int OFF_DO = OFF_Q + 2 * TILE_BYTES;  // 2 slots
  static constexpr int OFF_DS = OFF_DO + 2 * TILE_BYTES;
  static constexpr int OFF_STG = OFF_DS + (DS_ALIAS ? 0 : DS_BYTES);  // 4 warps x 2 buffers x 2 KB
  static constexpr int OFF_VEC = OFF_STG + 16384;  // 2 slots x (-LSE log2e, D) x 512 B
  static constexpr int OFF_BAR = OFF_VEC + 2048;
  static constexpr int NUM_BARS = 20;
  static constexpr int SMEM_BYTES = OFF_BAR + NUM_BARS * 8 + 16 + 1024;
  static constexpr uint32_t COL_S = 0;    // S^T; then per 64 queries: P^T bf16 in +[0,32)
  static constexpr uint32_t COL_DP = 128;  // dP^T; then per 64 queries: dS^T bf16 in +[0,32)
  static constexpr uint32_t COL_DV = 256;
  static constexpr uint32_t COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = (D == 64) ? 384 : 128;
  static constexpr bool DQ_SHARES_DP = (COL_DQ == COL_DP);
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct BwdBars {
  uint32_t base;
  __device__ uint32_t kv_full() const { return base; }
  __device__ uint32_t q_full(int s) const { return base + 8u * (1 + s); }
  __device__ uint32_t q_empty(int s) const { return base + 8u * (3 + s); }
  __device__ uint32_t do_full(int s) const { return base + 8u * (5 + s); }
  __device__ uint32_t do_empty(int s) const { return base + 8u * (7 + s); }
  __device__ uint32_t s_full() const { return base + 8u * 9; }
  __device__ uint32_t dp_full() const { return base + 8u * 10; }
  __device__ uint32_t p_ready() const { return base + 8u * 11; }
  __device__ uint32_t dst_ready() const { return base + 8u * 12; }  // dS^T in tensor memory
  __device__ uint32_t dss_ready() const { return base + 8u * 19; }  // dS in shared memory
  __device__ uint32_t dv_done() const { return base + 8u * 13; }
  __device__ uint32_t dq_full() const { return base + 8u * 14; }
  __device__ uint32_t dq_free() const { return base + 8u * 15; }
  __device__ uint32_t dkdv_done() const { return base + 8u * 16; }
  __device__ uint32_t epi() const { return base + 8u * 17; }
  __device__ uint32_t teardown() const { return base + 8u * 18; }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 100000000ull) break;  // 100 ms
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ------------------------------------------------------------------ preprocess
// D = rowsum(dO * O) and -LSE * log2(e) per query row (0 in the padding rows
// up to Npad), and zeros in the fp32 dQ accumulator. d/8 lanes per row, each
// covering 8 consecutive elements.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdParams p, long long total_rows) {
  const int lpr = p.d_pad >> 3;  // lanes per row (a power of two)
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gt / lpr;
  const int sub = static_cast<int>(gt - row * lpr);
  const bool valid = row < total_rows;
  const long long bh = valid ? row / p.Npad : 0;
  const int n = valid ? static_cast<int>(row - bh * p.Npad) : 0;
  // the row's sequence: fixed length N, or a packed batch's sequence b
  long long tok = 0;  // row index of [B*Hq, N] (fixed) or token index of [T, Hq] (packed)
  int len = p.N;
  if (p.cu_seqlens) {
    const int b = static_cast<int>(bh / p.Hq);
    const int s0 = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - s0;
    if (len < 0 || len > p.N || s0 < 0 || s0 + len > p.total) len = 0;  // reported by the main kernel
    tok = (static_cast<long long>(s0) + n) * p.Hq + (bh - static_cast<long long>(b) * p.Hq);
  } else {
    tok = bh * p.N + n;
  }
  const bool real = valid && n < len;
  const bool col = sub * 8 < p.d;
  // elements of O, dO and the dQ accumulator; rows of the LSE vector
  const long long elems = p.cu_seqlens ? static_cast<long long>(p.total) * p.Hq * p.d
                                       : total_rows / p.Npad * p.N * p.d;
  const long long lse_rows = p.cu_seqlens ? static_cast<long long>(p.total) * p.Hq : total_rows / p.Npad * p.N;
  float acc = 0.f;
  if (real && col && in_bounds(tok * p.d + sub * 8 + 7, elems, p.status, 0)) {
    const long long off = tok * p.d + sub * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(p.o + off);
    const uint4 gv = *reinterpret_cast<const uint4*>(p.dout + off);
    const uint32_t oa[4] = {ov.x, ov.y, ov.z, ov.w};
    const uint32_t ga[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) acc += bf16_lo(oa[e]) * bf16_lo(ga[e]) + bf16_hi(oa[e]) * bf16_hi(ga[e]);
    float4* z = reinterpret_cast<float4*>(p.dq_accum + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int off = lpr >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (valid && sub == 0 && in_bounds(row, total_rows, p.status, 1)) {
    p.delta[row] = real ? acc : 0.f;
    const long long lse_i = p.cu_seqlens ? (bh - (bh / p.Hq) * p.Hq) * p.total + (tok / p.Hq) : bh * p.N + n;
    p.neg_lse2[row] = real && in_bounds(lse_i, lse_rows, p.status, 2) ? -p.lse[lse_i] * LOG2E : 0.f;
  }
}

// ----------------------------------------------------------------- postprocess
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                                       long long n8, float scale) {
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * t];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * t + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x * scale, a.y * scale);
    o.y = pack_bf16x2(a.z * scale, a.w * scale);
    o.z = pack_bf16x2(b.x * scale, b.y * scale);
    o.w = pack_bf16x2(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[t] = o;
  }
}

// ------------------------------------------------------------------ main kernel
// (query head in the GQA group, query tile) of successive loop iterations:
// the tile runs first..last-1, then the next head starts again at first.
struct QWalk {
  int head, tile, first, last;
  __device__ QWalk(int first_tile, int num_tiles) : head(0), tile(first_tile), first(first_tile), last(num_tiles) {}
  __device__ void next() {
    if (++tile == last) {
      tile = first;
      ++head;
    }
  }
};

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                    const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1-D grid, head-major: all key tiles of one KV head back to back (the
  // longest causal loops first), so resident CTAs share a few heads' Q, dO
  // and dQ accumulator in L2.
  const int bkv = static_cast<int>(blockIdx.x) / p.num_tiles;  // b * Hkv + kvh
  const int j = static_cast<int>(blockIdx.x) - bkv * p.num_tiles;  // key tile
  const int b = bkv / p.Hkv;
  const int kvh = bkv - b * p.Hkv;
  // A packed batch's sequence b: tokens s0 .. s0 + len - 1. CTAs whose key
  // tile lies past the sequence's end leave at once.
  int s0 = 0, len = p.N;
  if (VARLEN) {
    s0 = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - s0;
    if (len < 0 || len > p.N || s0 < 0 || s0 + len > p.total) {
      if (threadIdx.x == 0 && j == 0) report_status(p.status, FA_ERR_INVALID_ARG | (SITE_SEQLENS << 8));
      return;
    }
  }
  const int T = VARLEN ? (len + BT - 1) / BT : p.num_tiles;
  if (VARLEN && j >= T) return;
  const int i0 = CAUSAL ? j : 0;
  const int nq = T - i0;
  const int n_it = p.group * nq;
  // TMA coordinates of 128 rows starting at row r of a head (fixed: y = row,
  // z = head; packed: y = head, z = token)
  auto tma_rows = [&](uint32_t dst, const CUtensorMap* m, uint32_t bar, int x, int r, int head) {
    if (VARLEN)
      tma_load_3d(dst, m, bar, x, head, s0 + r);
    else
      tma_load_3d(dst, m, bar, x, r, head);
  };
  const int kv_head = VARLEN ? kvh : bkv;  // K, V, dK, dV map head coordinate

  const BwdBars bars{base + C::OFF_BAR};
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + C::NUM_BARS * 8);
  volatile int* const abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    mbar_init(bars.kv_full(), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bars.q_full(s), 1);
      mbar_init(bars.q_empty(s), 1);
      mbar_init(bars.do_full(s), 1);
      mbar_init(bars.do_empty(s), 1);
    }
    mbar_init(bars.s_full(), 1);
    mbar_init(bars.dp_full(), 1);
    mbar_init(bars.p_ready(), 8);  // one arrive per compute warp (two warpgroups)
    mbar_init(bars.dst_ready(), 8);
    mbar_init(bars.dss_ready(), 8);
    mbar_init(bars.dv_done(), 1);
    mbar_init(bars.dq_full(), 1);
    mbar_init(bars.dq_free(), 4);
    mbar_init(bars.dkdv_done(), 1);
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
    prefetch_tmap(&tmdO);
    prefetch_tmap(&tmdQacc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Iteration it visits query head (it / nq) of the group and query tile
  // i0 + it % nq. Each role walks these in order with a QWalk (no division).
  const int bhq0 = b * p.Hq + kvh * p.group;  // first query head of the group, as b * Hq + hq
  const int qhead0 = VARLEN ? kvh * p.group : bhq0;  // its Q, dO, dQ map head coordinate
  auto ds_smem = [&](int st) -> uint32_t {
    return C::DS_ALIAS ? base + C::OFF_DO + st * C::TILE_BYTES : base + C::OFF_DS;
  };

  if (warp >= 12) {
    // warpgroup 3: producer, MMA issuer and two warps without a role
    setmaxnreg_dec<REGS_OTHER>();
    if (warp == PRODUCER_WARP) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        mbar_arrive_expect_tx(bars.kv_full(), 2 * C::TILE_BYTES);
        for (int bx = 0; bx < C::BOXES; ++bx) {
          tma_rows(base + C::OFF_K + bx * C::BOX_BYTES, &tmK, bars.kv_full(), bx * 64, j * BT, kv_head);
          tma_rows(base + C::OFF_V + bx * C::BOX_BYTES, &tmV, bars.kv_full(), bx * 64, j * BT, kv_head);
        }
        int issued = 0;
        QWalk qw(i0, T);
        for (int it = 0; it < n_it; ++it, qw.next()) {
          const int st = it & 1;
          const uint32_t ph = (it >> 1) & 1;
          const int bhq = bhq0 + qw.head;
          const int qh = qhead0 + qw.head;
          const int i = qw.tile;
          if (!mbar_wait_sleep(bars.q_empty(st), ph ^ 1, abort, p.status, SITE_BWD + 1)) break;
          mbar_arrive_expect_tx(bars.q_full(st), C::TILE_BYTES + 1024);
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_rows(base + C::OFF_Q + st * C::TILE_BYTES + bx * C::BOX_BYTES, &tmQ, bars.q_full(st), bx * 64,
                     i * BT, qh);
          const long long voff = static_cast<long long>(bhq) * p.Npad + i * BT;
          bulk_load_1d(base + C::OFF_VEC + st * 1024, p.neg_lse2 + voff, 512, bars.q_full(st));
          bulk_load_1d(base + C::OFF_VEC + st * 1024 + 512, p.delta + voff, 512, bars.q_full(st));
          if (!mbar_wait_sleep(bars.do_empty(st), ph ^ 1, abort, p.status, SITE_BWD + 2)) {
            issued = 2 * it + 1;
            break;
          }
          mbar_arrive_expect_tx(bars.do_full(st), C::TILE_BYTES);
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_rows(base + C::OFF_DO + st * C::TILE_BYTES + bx * C::BOX_BYTES, &tmdO, bars.do_full(st), bx * 64,
                     i * BT, qh);
          issued = 2 * it + 2;
        }
        if (*abort) {
          drain_wait(bars.kv_full(), 0);
          for (int t = (issued > 4 ? issued - 4 : 0); t < issued; ++t) {
            const int it = t >> 1;
            const uint32_t bar = (t & 1) ? bars.do_full(it & 1) : bars.q_full(it & 1);
            drain_wait(bar, (it >> 1) & 1);
          }
        }
      }
    } else if (warp == MMA_WARP) {
      // ------------------------------------------------------------ MMA issue
      if (lane == 0) {
        constexpr uint32_t IDESC_SS = idesc_bf16(BT, BT, false, false);
        constexpr uint32_t IDESC_TS = idesc_bf16(BT, D, false, true);
        constexpr uint32_t IDESC_DQ = idesc_bf16(BT, D, true, true);
        const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V;
        // K and V stay put for the whole CTA: their descriptors are fixed
        const uint64_t dk_ss = smem_desc_sw128(sK, 16, 1024), dv_ss = smem_desc_sw128(sV, 16, 1024);
        const uint64_t dk_mn = smem_desc_sw128(sK, C::BOX_BYTES, 1024);
        auto issue_st = [&](int it) {  // S^T = K_j Q_i^T into the S^T columns
          const uint64_t dq = smem_desc_sw128(base + C::OFF_Q + (it & 1) * C::TILE_BYTES, 16, 1024);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
            mma_ss(tmem + C::COL_S, desc_plus(dk_ss, off), desc_plus(dq, off), IDESC_SS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bars.s_full());
        };
        bool ok = mbar_wait_sleep(bars.kv_full(), 0, abort, p.status, SITE_BWD + 3) &&
                  mbar_wait_sleep(bars.q_full(0), 0, abort, p.status, SITE_BWD + 4);
        if (ok) {
          tc_fence_after();
          issue_st(0);
        }
        // Per iteration: dP^T(it), dV(it), S^T(it + 1), dK(it), dQ(it). S^T(it + 1)
        // goes into the S^T columns as soon as dV(it) has read P^T(it) from
        // them (tcgen05 MMAs of one thread run in issue order), so the compute
        // warps form P^T(it + 1) while the pipe runs dK(it) and dQ(it).
        for (int it = 0; ok && it < n_it; ++it) {
          const int st = it & 1;
          const uint32_t ph = (it >> 1) & 1;
          const uint32_t sQ = base + C::OFF_Q + st * C::TILE_BYTES;
          const uint32_t sdO = base + C::OFF_DO + st * C::TILE_BYTES;
          if (!mbar_wait_sleep(bars.do_full(st), ph, abort, p.status, SITE_BWD + 5)) break;
          if (C::DQ_SHARES_DP && it > 0 && !mbar_wait_sleep(bars.dq_free(), (it - 1) & 1, abort, p.status, SITE_BWD + 6))
            break;
          tc_fence_after();
          const uint64_t ddo = smem_desc_sw128(sdO, 16, 1024), ddo_mn = smem_desc_sw128(sdO, C::BOX_BYTES, 1024);
          const uint64_t dq_mn = smem_desc_sw128(sQ, C::BOX_BYTES, 1024);
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // dP^T = V_j dO_i^T
            const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
            mma_ss(tmem + C::COL_DP, desc_plus(dv_ss, off), desc_plus(ddo, off), IDESC_SS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bars.dp_full());
          if (!mbar_wait_sleep(bars.p_ready(), it & 1, abort, p.status, SITE_BWD + 7)) break;
          tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)  // dV += P^T dO_i
            mma_ts(tmem + C::COL_DV, tmem + C::COL_S + (kk >> 2) * 64 + (kk & 3) * 8, desc_plus(ddo_mn, kk * 2048),
                   IDESC_TS, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bars.dv_done());
          if (it + 1 < n_it) {
            if (!mbar_wait_sleep(bars.q_full(st ^ 1), ((it + 1) >> 1) & 1, abort, p.status, SITE_BWD + 4)) break;
            tc_fence_after();
            issue_st(it + 1);
          }
          if (!mbar_wait_sleep(bars.dst_ready(), it & 1, abort, p.status, SITE_BWD + 8)) break;
          tc_fence_after();
  #pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)  // dK += dS^T Q_i (dS^T over the dP^T columns)
            mma_ts(tmem + C::COL_DK, tmem + C::COL_DP + (kk >> 2) * 64 + (kk & 3) * 8, desc_plus(dq_mn, kk * 2048),
                   IDESC_TS, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bars.q_empty(st));
          if (!mbar_wait_sleep(bars.dss_ready(), it & 1, abort, p.status, SITE_BWD + 16)) break;
          if (!C::DQ_SHARES_DP && it > 0 &&
              !mbar_wait_sleep(bars.dq_free(), (it - 1) & 1, abort, p.status, SITE_BWD + 6))
            break;
          tc_fence_after();
          const uint64_t dds = smem_desc_sw128(ds_smem(st), 16384, 1024);
  #pragma unroll
          for (int kk = 0; kk < BT / 16; ++kk)  // dQ_i = dS K_j (A and B MN-major)
            mma_ss(tmem + C::COL_DQ, desc_plus(dds, kk * 2048), desc_plus(dk_mn, kk * 2048), IDESC_DQ,
                   kk > 0 ? 1u : 0u);
          mma_commit(bars.dq_full());
          mma_commit(bars.do_empty(st));
        }
        mma_commit(bars.dkdv_done());
      }
    }  // warps 14, 15: no role
  } else if (warp < 8) {
    // ------------------------------------------------------------ P and dS (thread = key row)
    // warpgroups 0 and 1, 64 query columns each
    setmaxnreg_inc<REGS_COMPUTE>();
    const int half = warp >> 2;  // query columns [64 half, 64 half + 64) of S^T and dP^T
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S + 64 * half;  // S^T; then P^T at +0
    const uint32_t tDP = tmem + lane_off + C::COL_DP + 64 * half;  // dP^T; then dS^T at +0
    const float cl2 = p.scale_log2;
    bool ok = true;
    QWalk qw(i0, T);
    for (int it = 0; ok && it < n_it; ++it, qw.next()) {
      const int st = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      const int i = qw.tile;
      ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.q_full(st), ph, abort, p.status, SITE_BWD + 9));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.s_full(), it & 1, abort, p.status, SITE_BWD + 10));
      if (!ok) break;
      tc_fence_after();
      const float* vec = reinterpret_cast<const float*>(base_ptr + C::OFF_VEC + st * 1024);
      const float* vec_lse = vec + 64 * half;
      const float* vec_d = vec + 128 + 64 * half;
      const int qlim = len - i * BT - 64 * half;  // queries of this half past the end are padding
      // a packed batch's keys past the sequence's end (the next sequence's
      // tokens in the tile) take no part: P^T = 0 keeps them out of dS and dQ
      const bool key_out = VARLEN && j * BT + r >= len;
      uint32_t pk[32];  // P^T of this half, bf16 pairs: kept for dS
      {
        float s[64];
        {
          uint32_t t[2][32];
          tmem_ld_x32(tS, t[0]);
          tmem_ld_x32(tS + 32, t[1]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(t[c][e]);
        }
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(vec_lse + c);
          s[c] = ex2(fmaf(s[c], cl2, l4.x));
          s[c + 1] = ex2(fmaf(s[c + 1], cl2, l4.y));
          s[c + 2] = ex2(fmaf(s[c + 2], cl2, l4.z));
          s[c + 3] = ex2(fmaf(s[c + 3], cl2, l4.w));
        }
        if (CAUSAL && i == j) {  // diagonal tile: key r sees queries >= r
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (64 * half + c < r) s[c] = 0.f;
        }
        if (qlim < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= qlim) s[c] = 0.f;
        }
        if (key_out) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(s[2 * e], s[2 * e + 1]);
        tmem_st_x16(tS, *reinterpret_cast<const uint32_t(*)[16]>(pk));
        tmem_st_x16(tS + 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + 16));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.p_ready());

      ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.dp_full(), it & 1, abort, p.status, SITE_BWD + 11));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - D), 32 queries at a time with P^T from registers (the S^T
      // columns already hold the next S^T once dV has read P^T): into tensor
      // memory over the first 32 of this warpgroup's 64 dP^T columns (each
      // 16-column chunk is written only after the 32 columns it covers have
      // been read), so dK can start at once, then into shared memory once dV
      // has finished reading this dO slot (dQ)
      uint32_t dsk[32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t t[32];
        tmem_ld_x32(tDP + cc * 32, t);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = cc * 32 + 2 * e;
          const uint32_t pp = pk[cc * 16 + e];
          const float2 dd = *reinterpret_cast<const float2*>(vec_d + c);
          dsk[cc * 16 + e] = pack_bf16x2(bf16_lo(pp) * (__uint_as_float(t[2 * e]) - dd.x),
                                         bf16_hi(pp) * (__uint_as_float(t[2 * e + 1]) - dd.y));
        }
        tmem_st_x16(tDP + cc * 16, *reinterpret_cast<const uint32_t(*)[16]>(dsk + cc * 16));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.dst_ready());
      ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.dv_done(), it & 1, abort, p.status, SITE_BWD + 12));
      if (!ok) break;
      const uint32_t box = ds_smem(st) + half * C::BOX_BYTES;  // queries [64 half, 64 half + 64)
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t addr = box + sw128_offset(r, ch);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dsk[4 * ch]), "r"(dsk[4 * ch + 1]),
                     "r"(dsk[4 * ch + 2]), "r"(dsk[4 * ch + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.dss_ready());
    }
    // ------------------------------------------------------------ dK, dV epilogue
    if (half == 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.dkdv_done(), 0, abort, p.status, SITE_BWD + 13));
    if (half != 0) ok = false;  // warpgroup 0 writes dK and dV
    if (ok) {
      tc_fence_after();
      // A packed batch's last, partial key tile is written row by row: a
      // tile-wide store would reach into the next sequence's rows.
      const bool direct = VARLEN && (j + 1) * BT > len;
      for (int which = 0; which < 2; ++which) {
        const uint32_t src = tmem + lane_off + (which ? C::COL_DV : C::COL_DK);
        const float mul = which ? 1.0f : p.scale;
        const uint32_t stage = base + C::OFF_Q + which * C::TILE_BYTES;
        uint16_t* const grow = (which ? p.dv : p.dk) + (static_cast<size_t>(s0 + j * BT + r) * p.Hkv + kvh) * p.d;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t t[32];
          tmem_ld_x32(src + c, t);
          tmem_wait_ld();
          const uint32_t box = stage + (c >> 6) * C::BOX_BYTES;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = pack_bf16x2(__uint_as_float(t[q * 8 + 2 * e]) * mul, __uint_as_float(t[q * 8 + 2 * e + 1]) * mul);
            if (direct) {
              if (j * BT + r < len && c + q * 8 < p.d &&
                  in_bounds((grow - (which ? p.dv : p.dk)) + c + q * 8 + 7,
                            static_cast<long long>(p.total) * p.Hkv * p.d, p.status, 3))
                *reinterpret_cast<uint4*>(grow + c + q * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            } else {
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(box + sw128_offset(r, ((c & 63) >> 3) + q)),
                           "r"(w4[0]), "r"(w4[1]), "r"(w4[2]), "r"(w4[3])
                           : "memory");
            }
          }
        }
      }
      if (!direct) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars.epi());
        if (r == 0 && mbar_wait_sleep(bars.epi(), 0, abort, p.status, SITE_BWD + 14)) {
          for (int bx = 0; bx < C::BOXES; ++bx) {
            if (VARLEN) {
              tma_store_3d(&tmdK, base + C::OFF_Q + bx * C::BOX_BYTES, bx * 64, kvh, s0 + j * BT);
              tma_store_3d(&tmdV, base + C::OFF_Q + C::TILE_BYTES + bx * C::BOX_BYTES, bx * 64, kvh, s0 + j * BT);
            } else {
              tma_store_3d(&tmdK, base + C::OFF_Q + bx * C::BOX_BYTES, bx * 64, j * BT, bkv);
              tma_store_3d(&tmdV, base + C::OFF_Q + C::TILE_BYTES + bx * C::BOX_BYTES, bx * 64, j * BT, bkv);
            }
          }
          bulk_commit();
          bulk_wait_read0();
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ drain (thread = query row)
    // warpgroup 2
    setmaxnreg_inc<REGS_DRAIN>();
    const int w = warp & 3;
    const uint32_t tDQ = tmem + (static_cast<uint32_t>(w * 32) << 16) + C::COL_DQ;
    const uint32_t stg0 = base + C::OFF_STG + w * 2 * 2048;
    int cnt = 0;
    bool ok = true;
    QWalk qw(i0, T);
    for (int it = 0; ok && it < n_it; ++it) {
      const int qh = qhead0 + qw.head;
      const int row0 = qw.tile * BT + w * 32;
      qw.next();
      ok = __all_sync(0xffffffffu, mbar_wait_sleep(bars.dq_full(), it & 1, abort, p.status, SITE_BWD + 15));
      if (!ok) break;
      tc_fence_after();
      float acc[D];
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t t[32];
        tmem_ld_x32(tDQ + c, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[c + e] = __uint_as_float(t[e]);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.dq_free());
      if (row0 >= len) continue;  // every row of this warp is padding
      // (rows of a partial tile past the end carry dQ = 0 exactly, since their
      // P^T columns are 0: adding them into the next sequence's rows of a
      // packed batch changes nothing)
#pragma unroll
      for (int c16 = 0; c16 < D / 16; ++c16) {
        if (c16 * 16 >= p.d) break;  // zero-padded columns (d = 96)
        const uint32_t buf = stg0 + (cnt & 1) * 2048;
        if (lane == 0) bulk_wait_read<1>();  // the reduce that last read this buffer is done with it
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t addr = buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(acc[c16 * 16 + 4 * q]),
                       "f"(acc[c16 * 16 + 4 * q + 1]), "f"(acc[c16 * 16 + 4 * q + 2]), "f"(acc[c16 * 16 + 4 * q + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (VARLEN)
            tma_reduce_add_3d(&tmdQacc, buf, c16 * 16, qh, s0 + row0);
          else
            tma_reduce_add_3d(&tmdQacc, buf, c16 * 16, row0, qh);
          bulk_commit();
        }
        ++cnt;
      }
    }
    if (lane == 0) bulk_wait0();
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
cudaError_t launch_main(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                        const CUtensorMap& tmdO, const CUtensorMap& tmdK, const CUtensorMap& tmdV,
                        const CUtensorMap& tmdQacc, const BwdParams& p, int B, cudaStream_t stream) {
  using C = BwdCfg<D>;
  auto kern = bwd_bf16_kernel<D, CAUSAL, VARLEN>;
  // the setmaxnreg increases wait until the CTA's register pool has room:
  // make sure the compiled launch allocation covers the split
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa_attr;
    cudaError_t e0 = cudaFuncGetAttributes(&fa_attr, kern);
    if (e0 != cudaSuccess) return e0;
    regs = fa_attr.numRegs;
  }
  if (256 * REGS_COMPUTE + 128 * REGS_DRAIN + 128 * REGS_OTHER > BWD_THREADS * regs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(B * p.Hkv * p.num_tiles);
  kern<<<grid, BWD_THREADS, C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_main_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          const CUtensorMap& tmdO, const CUtensorMap& tmdK, const CUtensorMap& tmdV,
                          const CUtensorMap& tmdQacc, const BwdParams& p, int B, bool causal, cudaStream_t stream) {
  if (p.cu_seqlens)
    return causal ? launch_main<D, true, true>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, stream)
                  : launch_main<D, false, true>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, stream);
  return causal ? launch_main<D, true, false>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, stream)
                : launch_main<D, false, false>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, stream);
}

}  // namespace

cudaError_t launch_bwd_bf16(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmdO, const CUtensorMap& tmdK, const CUtensorMap& tmdV,
                            const CUtensorMap& tmdQacc, const BwdParams& p, int B, bool causal,
                            cudaStream_t stream) {
  const long long BH = static_cast<long long>(B) * p.Hq;
  const long long rows = BH * p.Npad;
  const long long threads = rows * (p.d_pad / 8);
  bwd_pre_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(p, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.d_pad == 64)
    e = launch_main_d<64>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, causal, stream);
  else
    e = launch_main_d<128>(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmdQacc, p, B, causal, stream);
  if (e != cudaSuccess) return e;
  // dQ = scale * accumulator over every element of dQ's layout
  const long long elems = p.cu_seqlens ? static_cast<long long>(p.total) * p.Hq * p.d : BH * p.N * p.d;
  const long long n8 = elems / 8;
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  bwd_post_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p.dq_accum, p.dq, n8, p.scale);
  return cudaGetLastError();
}

}  // namespace fa
