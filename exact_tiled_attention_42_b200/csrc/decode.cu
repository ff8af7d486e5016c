// Decode-shaped forward: a few query rows per head against a long key
// sequence (Nq << Nk), the case of generating with a key/value cache.
//
// The attention is the one the other kernels compute ("FlashAttention: The
// Algorithm That Made Long-Context AI Possible", sections "The quadratic
// bottleneck in standard attention" and "What tiling changes"), with the
// queries taken as the last Nq positions of the sequence for the causal mask.
// Each key and value is read once and used by only g * Nq query rows, so the
// kernel is bound by HBM bandwidth: what matters is keeping bytes in flight on
// every SM and spending little shared-memory bandwidth per byte. The key
// dimension is split across CTAs (one CTA per KV head and key chunk, so the g
// query heads of a GQA group share each K/V tile); each CTA streams its chunk
// through a 3-stage TMA ring (two CTAs per SM) and keeps a running max and sum
// per query row; a second kernel merges the chunks by log-sum-exp.
//
// The query rows of a KV head (at most 16) form the M = 16 side of warp-level
// bf16 MMAs (mma.sync m16n8k16, fp32 accumulate): the products are tiny dense
// contractions and the fragments come straight from the swizzled TMA tiles
// with ldmatrix, so shared memory is read about once per byte. Per 64-key tile
// (8 warps):
//   S = Q K^T  warp w: keys 8w..8w+7, all of d (Q fragments stay in registers)
//   softmax    warp w: rows 2w, 2w+1 (two keys per lane), P (bf16) to smem
//   O += P V   warp w: output columns 16w.. (d = 128) or 8w.. (d = 64)
#include "common.cuh"
#include "kernels.h"

namespace fa {
namespace {

constexpr int KT = 64;        // keys per tile
constexpr int NSTAGE = 3;     // tiles in flight per CTA (two CTAs fit on an SM)
constexpr int THREADS = 256;
constexpr int MR = 16;        // MMA rows: query rows of a KV head, padded
constexpr int SS = KT + 4;    // fp32 score row stride (words)
constexpr int PS = KT + 8;    // bf16 P row stride (elements): 144 B rows keep ldmatrix conflict-free
constexpr float LN2 = 0.69314718055994530942f;

template <int D>
struct DecCfg {
  static constexpr int BOX = KT * 128;          // 64 keys x 64 bf16 (128 B rows)
  static constexpr int TILE = (D / 64) * BOX;   // one K or V tile
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = NSTAGE * TILE;
  static constexpr int OFF_S = 2 * NSTAGE * TILE;           // fp32 [MR][SS]
  static constexpr int OFF_P = OFF_S + MR * SS * 4;         // bf16 [MR][PS]
  static constexpr int OFF_A = OFF_P + MR * PS * 2;         // fp32 [MR] rescale, then 1 / l
  static constexpr int OFF_BAR = OFF_A + MR * 4;
  static constexpr int SMEM = OFF_BAR + NSTAGE * 8 + 8 + 1024;
  static constexpr int NB = D / 64;                         // 8-column blocks per warp in P V
};

// Byte offset of element (row, col) in a tile of 64-row, 128B-swizzled boxes.
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
  return (col >> 6) * (KT * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}

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
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
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
__global__ void __launch_bounds__(THREADS, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const bp = smem_raw + (base - raw);
  float* const ssc = reinterpret_cast<float*>(bp + C::OFF_S);
  uint16_t* const sp = reinterpret_cast<uint16_t*>(bp + C::OFF_P);
  float* const salpha = reinterpret_cast<float*>(bp + C::OFF_A);
  volatile int* const abort = reinterpret_cast<volatile int*>(bp + C::OFF_BAR + NSTAGE * 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;  // mma fragment row group and column pair

  const int bkv = static_cast<int>(blockIdx.x) / p.splits;  // b * Hkv + kvh
  const int split = static_cast<int>(blockIdx.x) - bkv * p.splits;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.Nk, k_begin + p.keys_per_split);
  const int ntiles = k_end > k_begin ? (k_end - k_begin + KT - 1) / KT : 0;
  const int R = p.R;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(base + C::OFF_BAR + 8 * s, 1);
    *abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int t) {
    const int s = t % NSTAGE;
    const uint32_t bar = base + C::OFF_BAR + 8 * s;
    mbar_arrive_expect_tx(bar, 2 * C::TILE);
    for (int bx = 0; bx < D / 64; ++bx) {
      tma_load_3d(base + C::OFF_K + s * C::TILE + bx * C::BOX, &tmK, bar, bx * 64, k_begin + t * KT, bkv);
      tma_load_3d(base + C::OFF_V + s * C::TILE + bx * C::BOX, &tmV, bar, bx * 64, k_begin + t * KT, bkv);
    }
  };
  if (tid == 0)
    for (int t = 0; t < ntiles && t < NSTAGE - 1; ++t) issue(t);

  // Q fragments (A operand, rows = query rows of this KV head, k = d), kept in
  // registers: row r = (head in group) * Nq + query index; rows >= R are 0.
  uint32_t qa[D / 16][4];
  {
    auto qword = [&](int r, int c) -> uint32_t {  // bf16 pair (c, c + 1) of row r
      if (r >= R) return 0u;
      const int hq = kvh * p.group + r / p.Nq, qi = r % p.Nq;
      return *reinterpret_cast<const uint32_t*>(p.q + ((static_cast<long long>(b) * p.Hq + hq) * p.Nq + qi) * D + c);
    };
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa[ks][0] = qword(g4, 16 * ks + 2 * t4);
      qa[ks][1] = qword(g4 + 8, 16 * ks + 2 * t4);
      qa[ks][2] = qword(g4, 16 * ks + 8 + 2 * t4);
      qa[ks][3] = qword(g4 + 8, 16 * ks + 8 + 2 * t4);
    }
  }
  // query position in the sequence of fragment rows g4 and g4 + 8 (causal mask)
  const int qpos0 = (g4 % p.Nq) + p.Nk - p.Nq, qpos1 = ((g4 + 8) % p.Nq) + p.Nk - p.Nq;

  // running max / sum of the two rows this warp owns in the softmax
  float m_row[2] = {-INFINITY, -INFINITY}, l_row[2] = {0.f, 0.f};
  // P V accumulators: rows g4, g4 + 8; columns of this warp's NB 8-column blocks
  float acc[C::NB][4];
#pragma unroll
  for (int nb = 0; nb < C::NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
  int t_stop = ntiles;  // first tile not consumed (set on abort)

  for (int t = 0; t < ntiles; ++t) {
    const int s = t % NSTAGE;
    if (tid == 0 && t + NSTAGE - 1 < ntiles) issue(t + NSTAGE - 1);  // its stage was released at the end of t-1
    const bool got = mbar_wait(base + C::OFF_BAR + 8 * s, (t / NSTAGE) & 1, abort, p.status, SITE_BWD + 20);
    if (__syncthreads_or(!got)) {
      t_stop = t;
      break;
    }
    const uint32_t kt = base + C::OFF_K + s * C::TILE;
    const uint32_t vt = base + C::OFF_V + s * C::TILE;
    const int kt0 = k_begin + t * KT;
    // ---- S = Q K^T for keys 8w .. 8w + 7
    {
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3, ri = lane & 7;  // ldmatrix: matrix and row this lane addresses
#pragma unroll
      for (int ks = 0; ks < D / 16; ks += 2) {
        uint32_t b0, b1, b2, b3;  // (k-step ks: d 0-7, 8-15), (k-step ks + 1: d 0-7, 8-15)
        ldsm_x4(kt + tile_off(8 * warp + ri, 16 * ks + 8 * mi), b0, b1, b2, b3);
        mma16816(sc, qa[ks], b0, b1);
        mma16816(sc, qa[ks + 1], b2, b3);
      }
      const int key0 = kt0 + 8 * warp + 2 * t4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kg = key0 + (e & 1);
        const int qpos = e < 2 ? qpos0 : qpos1;
        const bool vis = kg < k_end && (!p.causal || kg <= qpos);
        ssc[(g4 + 8 * (e >> 1)) * SS + 8 * warp + 2 * t4 + (e & 1)] = vis ? sc[e] * p.scale_log2 : -INFINITY;
      }
    }
    __syncthreads();
    // ---- softmax: warp w takes rows 2w and 2w + 1 (rows >= R get P = 0)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = 2 * warp + h;
      float p0 = 0.f, p1 = 0.f;
      if (r < R) {
        const float s0 = ssc[r * SS + lane], s1 = ssc[r * SS + lane + 32];
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_row[h], mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = m_row[h] == -INFINITY ? 0.f : ex2(m_row[h] - m_use);
        p0 = ex2(s0 - m_use);
        p1 = ex2(s1 - m_use);
        float sum = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        l_row[h] = l_row[h] * alpha + sum;
        m_row[h] = m_new;
        if (lane == 0) salpha[r] = alpha;
      } else if (lane == 0) {
        salpha[r] = 0.f;
      }
      const uint32_t w01 = pack_bf16x2(p0, p1);
      sp[r * PS + lane] = static_cast<uint16_t>(w01 & 0xFFFFu);
      sp[r * PS + lane + 32] = static_cast<uint16_t>(w01 >> 16);
    }
    __syncthreads();
    // ---- O += P V for this warp's columns
    {
      const float a0 = salpha[g4], a1 = salpha[g4 + 8];
#pragma unroll
      for (int nb = 0; nb < C::NB; ++nb) {
        acc[nb][0] *= a0;
        acc[nb][1] *= a0;
        acc[nb][2] *= a1;
        acc[nb][3] *= a1;
      }
      const int mi = lane >> 3, ri = lane & 7;
      const uint32_t pbase = smem_u32(sp);
#pragma unroll
      for (int ks = 0; ks < KT / 16; ++ks) {
        uint32_t pa[4];  // A: rows 0-7 / 8-15 x keys 16ks + 0-7 / 8-15
        ldsm_x4(pbase + (((mi & 1) * 8 + ri) * PS + 16 * ks + (mi >> 1) * 8) * 2, pa[0], pa[1], pa[2], pa[3]);
        const int col0 = C::NB * 8 * warp;
        if (C::NB == 2) {
          uint32_t b0, b1, b2, b3;  // (keys 0-7, 8-15) x (columns col0.., col0 + 8..)
          ldsm_x4_t(vt + tile_off(16 * ks + (mi & 1) * 8 + ri, col0 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma16816(acc[0], pa, b0, b1);
          mma16816(acc[C::NB - 1], pa, b2, b3);
        } else {
          uint32_t b0, b1;
          ldsm_x2_t(vt + tile_off(16 * ks + (mi & 1) * 8 + ri, col0), b0, b1);
          mma16816(acc[0], pa, b0, b1);
        }
      }
    }
    __syncthreads();  // this stage, the scores and P are free again
  }

  // partial results of this split, normalised within the split
  if (t_stop == ntiles) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = 2 * warp + h;
      if (r < R && lane == 0) {
        salpha[r] = l_row[h] > 0.f ? 1.0f / l_row[h] : 0.f;
        p.lse_part[(static_cast<long long>(bkv) * p.splits + split) * R + r] =
            l_row[h] > 0.f ? (m_row[h] + __log2f(l_row[h])) * LN2 : -INFINITY;
      }
    }
    __syncthreads();
#pragma unroll
    for (int nb = 0; nb < C::NB; ++nb) {
      const int col = C::NB * 8 * warp + 8 * nb + 2 * t4;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = g4 + 8 * hh;
        if (r < R) {
          const float inv = salpha[r];
          float2 v2 = make_float2(acc[nb][2 * hh] * inv, acc[nb][2 * hh + 1] * inv);
          *reinterpret_cast<float2*>(p.o_part + ((static_cast<long long>(bkv) * p.splits + split) * R + r) * D + col) =
              v2;
        }
      }
    }
  } else if (tid == 0) {
    // let the copies still in flight (tiles t_stop .. t_stop + NSTAGE - 1) land
    // before the CTA exits; each wait is bounded
    for (int t = t_stop; t < ntiles && t < t_stop + NSTAGE; ++t) {
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(base + C::OFF_BAR + 8 * (t % NSTAGE), (t / NSTAGE) & 1))
        if (globaltimer() - t0 > 100000000ull) break;
    }
  }
}

// One warp per output row (b, hq, query): merge the splits by log-sum-exp.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecParams p, int rows) {
  const int w = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const int bh = w / p.Nq, qi = w - bh * p.Nq;
  const int b = bh / p.Hq, hq = bh - b * p.Hq;
  const int bkv = b * p.Hkv + hq / p.group;
  const int r = (hq % p.group) * p.Nq + qi;
  float mx = -INFINITY;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.lse_part[(static_cast<long long>(bkv) * p.splits + s) * p.R + r]);
  float wsum = 0.f;
  float o[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) o[e] = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const long long base_row = (static_cast<long long>(bkv) * p.splits + s) * p.R + r;
    const float l = p.lse_part[base_row];
    if (l == -INFINITY) continue;
    const float wgt = __expf(l - mx);
    wsum += wgt;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) o[e] = fmaf(wgt, p.o_part[base_row * D + lane + 32 * e], o[e]);
  }
  const float inv = 1.0f / wsum;
  const long long orow = static_cast<long long>(bh) * p.Nq + qi;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) {
    const float v = o[e] * inv;
    const uint32_t bits = __float_as_uint(v);
    p.o[orow * D + lane + 32 * e] = static_cast<uint16_t>((bits + 0x7FFFu + ((bits >> 16) & 1u)) >> 16);
  }
  if (lane == 0) p.lse[orow] = mx + __logf(wsum);
}

template <int D>
cudaError_t launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecParams& p, int B, cudaStream_t stream) {
  using C = DecCfg<D>;
  auto k1 = decode_split_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  k1<<<B * p.Hkv * p.splits, THREADS, C::SMEM, stream>>>(tmK, tmV, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = B * p.Hq * p.Nq;
  decode_combine_kernel<D><<<(rows * 32 + 255) / 256, 256, 0, stream>>>(p, rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecParams& p, int B, int d,
                          cudaStream_t stream) {
  return d == 64 ? launch<64>(tmK, tmV, p, B, stream) : launch<128>(tmK, tmV, p, B, stream);
}

}  // namespace fa
