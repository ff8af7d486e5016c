// Decode-shaped forward: a few query rows per head against a long key
// sequence (Nq << Nk), the case of generating with a key/value cache.
//
// The attention is the one the other kernels compute ("FlashAttention: The
// Algorithm That Made Long-Context AI Possible", sections "The quadratic
// bottleneck in standard attention" and "What tiling changes"), with the
// queries taken as the last Nq positions of the sequence for the causal mask.
// Each key and value is read once and used by only g * Nq query rows, so the
// kernel is bound by HBM bandwidth: what matters is keeping bytes in flight on
// every SM and spending little shared-memory bandwidth per byte.
//
// Work split. The work is a list of units (KV head, 64-key tile), head-major.
// The split pass runs as many CTAs as fit on the GPU at once (two per SM) and
// gives CTA c the contiguous units [c*U/G, (c+1)*U/G): every CTA streams the
// same number of tiles, whatever the number of heads or keys, and its TMA ring
// runs on across head boundaries. A CTA writes one partial result (rows
// normalised within its key range, plus their log-sum-exp) for each KV head it
// touches; the g query heads of a GQA group share each K/V tile. A second
// kernel merges the partials of a head by log-sum-exp.
//
// The query rows of a KV head (at most 16) form the M = 16 side of warp-level
// bf16 MMAs (mma.sync m16n8k16, fp32 accumulate): the products are tiny dense
// contractions, and the K and V fragments come straight from the swizzled TMA
// tiles with ldmatrix. One producer warp streams 64-key tiles of K and V
// through an mbarrier ring; each of the four consumer warps owns 16 keys of
// every tile and runs the whole tile step on its own, with no CTA barrier:
//   S = Q K^T   16 rows x 16 keys, Q fragments held in registers
//   softmax     running max and sum per row over the warp's keys; O rescaled
//               only when a max grows; P stays in registers, where the S
//               accumulator layout is already the A-operand layout of P V
//   O += P V    16 rows x d, fp32 in registers
// then frees the stage. When the CTA's range of a KV head ends, the four
// warps' (max, sum, O) are merged through the stage buffer they just read.

#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int KT = 64;        // keys per tile
constexpr int NCW = 4;        // consumer warps; warp w owns keys 16w .. 16w + 15 of every tile
constexpr int THREADS = (NCW + 1) * 32;  // + one producer warp
constexpr int MR = 16;        // MMA rows: query rows of a KV head, padded
constexpr float LN2 = 0.69314718055994530942f;

template <int D>
struct DecCfg {
  static constexpr int NSTAGE = D == 128 ? 3 : 4;    // tiles in flight per CTA
  static constexpr int MIN_CTAS = D == 128 ? 2 : 3;  // CTAs per SM the shared memory allows
  static constexpr int BOX = KT * 128;               // 64 keys x 64 bf16 (128 B rows)
  static constexpr int TILE = (D / 64) * BOX;        // one K or V tile
  static constexpr int STAGE = 2 * TILE;             // K then V; also holds the NCW x MR x D fp32 partials
  static constexpr int OFF_ML = NSTAGE * STAGE;      // fp32 [NCW][MR][2]: per-warp row max and sum
  static constexpr int OFF_BAR = OFF_ML + NCW * MR * 2 * 4;
  // barriers: full[NSTAGE], empty[NSTAGE], gather, combine; then the abort flag
  static constexpr int NBAR = 2 * NSTAGE + 2;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 8 + 1024;
  static_assert(NCW * MR * D * 4 == STAGE, "a stage holds the warps' partial outputs");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(THREADS, DecCfg<D>::MIN_CTAS)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecParams p) {
  using C = DecCfg<D>;
  constexpr int NST = C::NSTAGE;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const bp = smem_raw + (base - raw);
  float* const sml = reinterpret_cast<float*>(bp + C::OFF_ML);
  const uint32_t bar_full = base + C::OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * NST;
  const uint32_t bar_gather = bar_empty + 8 * NST;  // every warp has finished reading the stage
  const uint32_t bar_comb = bar_gather + 8;         // every warp's partial is in the stage
  volatile int* const abort = reinterpret_cast<volatile int*>(bp + C::OFF_BAR + C::NBAR * 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // this CTA's work units [u0, u0 + n): unit u = (KV head u / tiles, key tile u % tiles)
  const int cta = static_cast<int>(blockIdx.x);
  const long long u0 = static_cast<long long>(cta) * p.units / p.ctas;
  const int n = static_cast<int>(static_cast<long long>(cta + 1) * p.units / p.ctas - u0);

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, NCW);
    }
    mbar_init(bar_gather, NCW);
    mbar_init(bar_comb, NCW);
    *abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ---- producer: one thread streams K and V tiles through the ring
    if (lane != 0) return;
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    int issued = 0;
    int bkv = static_cast<int>(u0 / p.tiles);
    int t = static_cast<int>(u0 - static_cast<long long>(bkv) * p.tiles);
    for (int i = 0; i < n; ++i) {
      const int s = i % NST;
      // the producer waits most of the time: sleep rather than spin, so the
      // consumer warp that shares its scheduler keeps the issue slots
      if (i >= NST && !mbar_wait_sleep(bar_empty + 8 * s, ((i / NST) - 1) & 1, abort, p.status, SITE_BWD + 21))
        break;
      const uint32_t dst = base + s * C::STAGE;
      mbar_arrive_expect_tx(bar_full + 8 * s, 2 * C::TILE);
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d(dst + bx * C::BOX, &tmK, bar_full + 8 * s, bx * 64, t * KT, bkv);
        tma_load_3d(dst + C::TILE + bx * C::BOX, &tmV, bar_full + 8 * s, bx * 64, t * KT, bkv);
      }
      issued = i + 1;
      if (++t == p.tiles) {
        t = 0;
        ++bkv;
      }
    }
    // Stay until the last copies have landed (they may outlive the consumers
    // if those give up on a wait); each wait is bounded.
    for (int i = issued > NST ? issued - NST : 0; i < issued; ++i) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(bar_full + 8 * (i % NST), (i / NST) & 1))
        if (globaltimer() - t0 > 100000000ull) break;
    }
    return;
  }

  // ---- consumers: warp w owns keys 16w .. 16w + 15 of every tile and keeps
  // its own running max, sum and O for them; the warps' results for a KV head
  // are merged when the CTA's range of that head ends.
  const int g4 = lane >> 2, t4 = lane & 3;  // mma fragment row group and column pair
  const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const int R = p.R;
  const int kw = 16 * warp;
  // Keys visible to fragment rows g4 and g4 + 8 are those below lim0 / lim1:
  // Nk, or with the causal mask (query index r % Nq at sequence position
  // r % Nq + Nk - Nq) that position + 1. Computed once, without a division.
  int lim0 = p.Nk, lim1 = p.Nk;
  if (p.causal) {
    int q0 = g4, q1 = g4 + 8;
    while (q0 >= p.Nq) q0 -= p.Nq;
    while (q1 >= p.Nq) q1 -= p.Nq;
    lim0 = q0 + p.Nk - p.Nq + 1;
    lim1 = q1 + p.Nk - p.Nq + 1;
  }
  // Per-lane byte offsets of the ldmatrix rows in a 128B-swizzled 64-row box:
  // the 16-byte chunk index is XOR-ed with the row's low three bits, so the
  // k-step's chunk is applied below with one XOR. K: matrix mi holds keys
  // kw + 8 (mi >> 1) + ri at d chunk (mi & 1); V: keys kw + 8 (mi & 1) + ri at
  // column chunk (mi >> 1).
  const uint32_t lane_k = (kw + 8 * (mi >> 1) + ri) * 128 + (((ri ^ (mi & 1)) & 7) << 4);
  const uint32_t lane_v = (kw + 8 * (mi & 1) + ri) * 128 + (((ri ^ (mi >> 1)) & 7) << 4);

  uint32_t qa[D / 16][4];  // Q fragments of the current KV head (A operand, k = d)
  float m_r[2];            // running max of rows g4, g4 + 8 over this warp's keys (same across a quad)
  float l_r[2];            // this thread's share of the running sums
  float acc[D / 8][4];     // O rows g4, g4 + 8; columns 8 nb + 2 t4, + 1

  int bkv = static_cast<int>(u0 / p.tiles);
  int t = static_cast<int>(u0 - static_cast<long long>(bkv) * p.tiles);
  int nseg = 0;  // head ranges merged so far (phase of the gather / combine barriers)

  for (int i = 0; i < n; ++i) {
    const int s = i % NST;
    if (i == 0 || t == 0) {
      // a new KV head: its query rows. Row r = (head in group) * Nq + query
      // index, so the group's rows are consecutive in q from its first head's
      // first query (b * Hq + kvh * group) * Nq; rows >= R are 0.
      const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
      const uint16_t* const qg = p.q + ((static_cast<long long>(b) * p.Hq + kvh * p.group) * p.Nq) * D;
      auto qword = [&](int r, int c) -> uint32_t {  // bf16 pair (c, c + 1) of row r
        return r < R ? *reinterpret_cast<const uint32_t*>(qg + r * D + c) : 0u;
      };
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        qa[ks][0] = qword(g4, 16 * ks + 2 * t4);
        qa[ks][1] = qword(g4 + 8, 16 * ks + 2 * t4);
        qa[ks][2] = qword(g4, 16 * ks + 8 + 2 * t4);
        qa[ks][3] = qword(g4 + 8, 16 * ks + 8 + 2 * t4);
      }
      m_r[0] = m_r[1] = -INFINITY;
      l_r[0] = l_r[1] = 0.f;
#pragma unroll
      for (int nb = 0; nb < D / 8; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
    }
    if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar_full + 8 * s, (i / NST) & 1, abort, p.status, SITE_BWD + 22)))
      break;
    const uint32_t st = base + s * C::STAGE;  // K tile, then the V tile at + TILE

    // ---- S = Q K^T for this warp's keys (two 8-key blocks), base-2 scaled and masked
    float sc[2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t b0, b1, b2, b3;  // keys kw + 0-7: d lo, d hi; keys kw + 8-15: d lo, d hi
      ldsm_x4(st + (ks >> 2) * C::BOX + (lane_k ^ ((ks & 3) << 5)), b0, b1, b2, b3);
      mma16816(sc[0], qa[ks], b0, b1);
      mma16816(sc[1], qa[ks], b2, b3);
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
    {
      const int key0 = t * KT + kw + 2 * t4;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool vis = key0 + 8 * nb + (e & 1) < (e < 2 ? lim0 : lim1);
          sc[nb][e] = vis ? sc[nb][e] * p.scale_log2 : -INFINITY;
          if (e < 2) mx0 = fmaxf(mx0, sc[nb][e]);
          else mx1 = fmaxf(mx1, sc[nb][e]);
        }
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // ---- online softmax; O and the sums are rescaled only when a row's max grew
    {
      const float n0 = fmaxf(m_r[0], mx0), n1 = fmaxf(m_r[1], mx1);
      if (__any_sync(0xffffffffu, n0 > m_r[0] || n1 > m_r[1])) {
        const float a0 = m_r[0] == -INFINITY ? 0.f : ex2(m_r[0] - n0);
        const float a1 = m_r[1] == -INFINITY ? 0.f : ex2(m_r[1] - n1);
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb) {
          acc[nb][0] *= a0;
          acc[nb][1] *= a0;
          acc[nb][2] *= a1;
          acc[nb][3] *= a1;
        }
        l_r[0] *= a0;
        l_r[1] *= a1;
        m_r[0] = n0;
        m_r[1] = n1;
      }
    }
    uint32_t pa[4];  // P as the A operand of P V: rows g4 / g4 + 8, keys 2 t4 (+8)
    {
      const float mu0 = m_r[0] == -INFINITY ? 0.f : m_r[0];
      const float mu1 = m_r[1] == -INFINITY ? 0.f : m_r[1];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const float p0 = ex2(sc[nb][0] - mu0), p1 = ex2(sc[nb][1] - mu0);
        const float p2 = ex2(sc[nb][2] - mu1), p3 = ex2(sc[nb][3] - mu1);
        l_r[0] += p0 + p1;
        l_r[1] += p2 + p3;
        pa[2 * nb] = pack_bf16x2(p0, p1);
        pa[2 * nb + 1] = pack_bf16x2(p2, p3);
      }
    }
    // ---- O += P V over this warp's 16 keys, 16 columns per ldmatrix
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      uint32_t b0, b1, b2, b3;  // keys 0-7 / 8-15 of columns 16c + 0-7, then of 16c + 8-15
      ldsm_x4_t(st + C::TILE + (c >> 2) * C::BOX + (lane_v ^ ((c & 3) << 5)), b0, b1, b2, b3);
      mma16816(acc[2 * c], pa, b0, b1);
      mma16816(acc[2 * c + 1], pa, b2, b3);
    }

    if (i == n - 1 || t == p.tiles - 1) {
      // The CTA's range of this KV head ends. The warps' partial outputs go
      // into this stage (every warp has read it), then each thread merges a
      // share of the R x D output and writes the CTA's partial result to slot
      // cta + bkv, rows normalised within the range.
      float l0 = l_r[0], l1 = l_r[1];
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_gather);
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar_gather, nseg & 1, abort, p.status, SITE_BWD + 23))) break;
      float* const buf = reinterpret_cast<float*>(bp + s * C::STAGE);  // [NCW][MR][D]
#pragma unroll
      for (int nb = 0; nb < D / 8; ++nb) {
        *reinterpret_cast<float2*>(buf + (warp * MR + g4) * D + 8 * nb + 2 * t4) = make_float2(acc[nb][0], acc[nb][1]);
        *reinterpret_cast<float2*>(buf + (warp * MR + g4 + 8) * D + 8 * nb + 2 * t4) =
            make_float2(acc[nb][2], acc[nb][3]);
      }
      if (t4 == 0) {
        sml[(warp * MR + g4) * 2] = m_r[0];
        sml[(warp * MR + g4) * 2 + 1] = l0;
        sml[(warp * MR + g4 + 8) * 2] = m_r[1];
        sml[(warp * MR + g4 + 8) * 2 + 1] = l1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_comb);
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(bar_comb, nseg & 1, abort, p.status, SITE_BWD + 24))) break;
      ++nseg;
      const long long slot = static_cast<long long>(cta) + bkv;
      for (int idx = tid; idx < R * D; idx += NCW * 32) {
        const int r = idx / D, col = idx - r * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NCW; ++w) M = fmaxf(M, sml[(w * MR + r) * 2]);
        float L = 0.f, o = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NCW; ++w) {
            const float mw = sml[(w * MR + r) * 2];
            if (mw != -INFINITY) {
              const float f = ex2(mw - M);
              L = fmaf(f, sml[(w * MR + r) * 2 + 1], L);
              o = fmaf(f, buf[(w * MR + r) * D + col], o);
            }
          }
        }
        if (!in_bounds(slot * R + r, (p.ctas + p.units / p.tiles) * static_cast<long long>(R), p.status, 20)) continue;
        p.o_part[(slot * R + r) * D + col] = L > 0.f ? o / L : 0.f;
        if (col == 0) p.lse_part[slot * R + r] = L > 0.f ? (M + __log2f(L)) * LN2 : -INFINITY;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);  // this warp is done with the stage
    if (++t == p.tiles) {
      t = 0;
      ++bkv;
    }
  }
}

// One warp per output row (b, hq, query): merge the partial results of its KV
// head by log-sum-exp. The CTAs that touched head bkv are the owners of its
// first and last units; owner(u) = ((u + 1) * ctas - 1) / units.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecParams p, int rows) {
  const int w = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const int bh = w / p.Nq, qi = w - bh * p.Nq;
  const int b = bh / p.Hq, hq = bh - b * p.Hq;
  const int bkv = b * p.Hkv + hq / p.group;
  const int r = (hq % p.group) * p.Nq + qi;
  const long long first_unit = static_cast<long long>(bkv) * p.tiles;
  const long long c_first = ((first_unit + 1) * p.ctas - 1) / p.units;
  const long long c_last = ((first_unit + p.tiles) * p.ctas - 1) / p.units;
  const int nparts = static_cast<int>(c_last - c_first + 1);
  const long long slot0 = c_first + bkv;
  // every partial this row reads, and its output row, must lie in the buffers
  if (!in_bounds(slot0 + nparts - 1, p.ctas + p.units / p.tiles, p.status, 21) ||
      !in_bounds(static_cast<long long>(bh) * p.Nq + qi, p.units / p.tiles * p.group * p.Nq, p.status, 22))
    return;

  float mx = -INFINITY;
  for (int j = lane; j < nparts; j += 32) mx = fmaxf(mx, p.lse_part[(slot0 + j) * p.R + r]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float wsum = 0.f;
  float o[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) o[e] = 0.f;
  for (int j0 = 0; j0 < nparts; j0 += 32) {
    // lane j holds the weight of partial j0 + j
    float wl = 0.f;
    if (j0 + lane < nparts) {
      const float l = p.lse_part[(slot0 + j0 + lane) * p.R + r];
      wl = l == -INFINITY ? 0.f : __expf(l - mx);
    }
    wsum += wl;
    const int cnt = min(32, nparts - j0);
#pragma unroll 4
    for (int j = 0; j < cnt; ++j) {
      const float wgt = __shfl_sync(0xffffffffu, wl, j);
      const float* src = p.o_part + ((slot0 + j0 + j) * p.R + r) * D + lane;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) o[e] = fmaf(wgt, src[32 * e], o[e]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
  const float inv = 1.0f / wsum;
  const long long orow = static_cast<long long>(bh) * p.Nq + qi;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) {
    const uint32_t bits = __float_as_uint(o[e] * inv);
    p.o[orow * D + lane + 32 * e] = static_cast<uint16_t>((bits + 0x7FFFu + ((bits >> 16) & 1u)) >> 16);
  }
  if (lane == 0) p.lse[orow] = mx + __logf(wsum);
}

template <int D>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(decode_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<D>::SMEM);
}

template <int D>
cudaError_t launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecParams& p, int B, cudaStream_t stream) {
  cudaError_t e = set_smem<D>();
  if (e != cudaSuccess) return e;
  decode_split_kernel<D><<<p.ctas, THREADS, DecCfg<D>::SMEM, stream>>>(tmK, tmV, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = B * p.Hq * p.Nq;
  decode_combine_kernel<D><<<(rows * 32 + 255) / 256, 256, 0, stream>>>(p, rows);
  return cudaGetLastError();
}

template <int D>
int resident() {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (set_smem<D>() != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_split_kernel<D>, THREADS, DecCfg<D>::SMEM) !=
      cudaSuccess)
    return 0;
  return sms * per_sm;
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecParams& p, int B, int d,
                          cudaStream_t stream) {
  return d == 64 ? launch<64>(tmK, tmV, p, B, stream) : launch<128>(tmK, tmV, p, B, stream);
}

int decode_resident_ctas(int d) {
  // per device and head dimension, queried once (a racing first query just
  // stores the same value twice)
  static std::atomic<int> cache[64][2];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return d == 64 ? resident<64>() : resident<128>();
  std::atomic<int>& c = cache[dev][d == 64 ? 0 : 1];
  int v = c.load(std::memory_order_relaxed);
  if (v == 0) {
    v = d == 64 ? resident<64>() : resident<128>();
    c.store(v, std::memory_order_relaxed);
  }
  return v;
}

}  // namespace fa
