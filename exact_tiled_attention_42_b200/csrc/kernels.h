// Launchers shared between the kernel translation units and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace fa {

// Heads per group of the forward grid order: as many query heads as share
// about 32 MiB of K and V (a quarter of L2), all of them when that covers
// every head. Measured on B200 (forward, against heads fastest over all
// heads): long128, 4 MiB of bf16 K/V per head, groups of 8: DRAM traffic
// 608 -> 250 MB per launch, +3 %; gqa, groups of 32: +2 %; the FP8 workload,
// groups of 8: 488 -> 154 MB, +3 %; gpt2 causal (0.5 MiB per head, groups of
// 64): -3 % (groups of 8 there: -7 %, the causal tail).
inline int raster_heads_for(long long BH, int group, long long kv_bytes_per_kv_head) {
  const long long budget = 32ll << 20;
  const long long per_qhead = kv_bytes_per_kv_head / (group > 0 ? group : 1);
  long long G = per_qhead > 0 ? budget / per_qhead : BH;
  if (G < 1) G = 1;
  if (G > BH) G = BH;
  return static_cast<int>(G);
}

struct FwdParams {
  float* lse;        // [B*Hq, N]; packed batches: [Hq, T]
  int* status;       // device status word (bounded waits report here)
#ifdef FA_DEBUG_WITHHOLD
  int debug_withhold;  // debug build only: 1 = the producer never issues the first V tile
#endif
  // Packed variable-length batches only (null otherwise): sequence b owns
  // tokens cu_seqlens[b] .. cu_seqlens[b+1]-1 of the token-major [T, H, d]
  // tensors, and N is the largest sequence length the grid was sized for.
  const int* cu_seqlens;
  uint16_t* o;       // packed batches: O [T, Hq, d] for the per-thread stores of partial tiles
  int total;         // packed batches: T
  int d;             // head dimension of the tensors (96 runs on the 128-column tiles, zero-padded)
  int N;
  int Hq;
  int Hkv;
  int group;         // Hq / Hkv
  int num_qtiles;    // ceil(N / 128)
  int num_pairs;     // ceil(num_qtiles / 2): one CTA per pair of query tiles
  int raster_heads;  // heads per group of the grid order (raster_heads_for)
  float scale_log2;  // scale * log2(e)
};

// tmQ/tmO: bf16 [B*Hq, N, d]; tmK/tmV: bf16 [B*Hkv, N, d]; all with
// 64-column x 128-row boxes and 128-byte swizzle. Packed batches
// (p.cu_seqlens set): tmQ/tmO over [T, Hq, d], tmK/tmV over [T, Hkv, d]
// with 64-column x 1-head x 128-token boxes. d = 96 uses the d = 128 kernel:
// the maps' inner extent is 96, so loads fill columns 96..127 with zeros and
// stores clip them.
cudaError_t launch_fwd_bf16(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmO, const FwdParams& p, int BH, int d, bool causal,
                            cudaStream_t stream);

// Wide heads (d = 192, 256): one 128-row query tile per CTA and 64-key tiles
// (grid BH * p.num_qtiles). tmQ/tmO as for launch_fwd_bf16; tmK/tmV with
// 64-column x 64-row (packed: 64-token) boxes.
cudaError_t launch_fwd_wide(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmO, const FwdParams& p, int BH, int d, bool causal,
                            cudaStream_t stream);

struct BwdParams {
  const uint16_t* o;     // bf16 [B*Hq, N, d] (packed batches: [T, Hq, d])  (preprocess)
  const uint16_t* dout;  // bf16, as o                                      (preprocess)
  const float* lse;      // [B*Hq, N] (packed: [Hq, T]), natural log        (preprocess)
  float* delta;          // workspace [B*Hq, Npad]: D = rowsum(dO * O), 0 past each sequence's end
  float* neg_lse2;       // workspace [B*Hq, Npad]: -LSE * log2(e), 0 past each sequence's end
  float* dq_accum;       // workspace fp32, dQ's layout, zeroed by the preprocess
  uint16_t* dq;          // bf16, dQ's layout                               (postprocess)
  uint16_t* dk;          // packed batches: dK [T, Hkv, d] for the per-thread stores of partial tiles
  uint16_t* dv;          // packed batches: dV, as dk
  const int* cu_seqlens; // packed batches only (null otherwise): sequence offsets, B + 1 entries
  int* status;
  int total;             // packed batches: T
  int N;                 // sequence length (packed batches: the largest)
  int Npad;              // num_tiles * 128
  int Hq;
  int Hkv;
  int group;
  int num_tiles;         // ceil(N / 128): query tiles and key tiles
  int d;                 // head dimension of the tensors
  int d_pad;             // columns the kernel computes: 64 or 128 (d = 96 is zero-padded to 128)
  float scale;
  float scale_log2;
};

// Backward: preprocess (D, -LSE*log2 e, zero dq_accum), the main kernel over
// (key tile, KV head), and the dq postprocess. tmQ/tmdO: [B*Hq, N, d] bf16;
// tmK/tmV/tmdK/tmdV: [B*Hkv, N, d] bf16 (64 x 128 boxes, 128B swizzle);
// tmdQacc: fp32 [B*Hq, N, d] with 16 x 32 boxes and 64B swizzle. Packed
// batches (p.cu_seqlens set): the maps are over the token-major [T, H, d]
// tensors with 1-head boxes of the same shapes.
cudaError_t launch_bwd_bf16(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmdO, const CUtensorMap& tmdK, const CUtensorMap& tmdV,
                            const CUtensorMap& tmdQacc, const BwdParams& p, int B, bool causal,
                            cudaStream_t stream);

struct Fp8Params {
  // pre-pass
  const uint16_t* src[3];  // bf16 Q [B*Hq, N, d], K and V [B*Hkv, N, d]
  uint8_t* codes[3];       // e4m3 copies (Q and K rotated when rotate != 0)
  float* scales[3];        // one fp32 scale per 64-row block: [B*H, nblk]
  int heads[3];            // B*Hq, B*Hkv, B*Hkv
  uint64_t rotation_seed;
  int rotate;
  // forward
  float* lse;              // [B*Hq, N]
  int* status;
  int N;
  int nblk;                // ceil(N / 64)
  int Hq;
  int Hkv;
  int group;
  int num_qtiles;
  int num_pairs;
  int raster_heads;        // heads per group of the grid order (raster_heads_for)
  float score_log2;        // scale * log2(e), divided by d when rotated
};

// Pre-pass (rotation + block quantisation of Q, K, V) then the FP8 forward.
// tmQ8/tmK8/tmV8: e4m3 [B*H, N, d] with 128 x 128 boxes and 128B swizzle;
// tmO: bf16 output map as for the bf16 forward.
cudaError_t launch_fp8_quant(const Fp8Params& p, cudaStream_t stream);
cudaError_t launch_fwd_fp8(const CUtensorMap& tmQ8, const CUtensorMap& tmK8, const CUtensorMap& tmV8,
                           const CUtensorMap& tmO, const Fp8Params& p, int BH, bool causal, cudaStream_t stream);

struct MxParams {
  // pre-pass
  const uint16_t* src[3];  // bf16 Q [B*Hq, N, d], K and V [B*Hkv, N, d]
  uint8_t* codes[3];       // e4m3 copies (Q and K rotated when rotate != 0), same layouts
  uint8_t* exps[3];        // E8M0 exponents (e + 127): Q [B*Hq, N, 4] and K [B*Hkv, N, 4] (one per
                           // 32 columns); V [B*Hkv, d, vexp_stride]: per column one 4-byte word per
                           // 96-key tile, bytes 0-2 its three 32-key blocks, byte 3 zero
  int heads[3];            // B*Hq, B*Hkv, B*Hkv
  uint64_t rotation_seed;
  int rotate;
  int fit;                 // 1: exponent one higher when amax's significand exceeds 1.75
  // forward
  float* lse;              // [B*Hq, N]
  int* status;
  int N;
  int num_ktiles;          // ceil(N / 96): the forward's key tiles
  int vexp_stride;         // 4 * num_ktiles: bytes of V's exponents per column
  int Hq;
  int Hkv;
  int group;
  int num_qtiles;
  int num_pairs;           // ceil(num_qtiles / 2): one CTA per pair of query tiles
  int raster_heads;        // heads per group of the grid order (raster_heads_for)
  float score_log2;        // scale * log2(e), divided by d when rotated
};

// MXFP8 pre-pass (rotation + MX quantisation of Q, K along d and of V along
// the keys) and the MXFP8 forward (d = 128; two query tiles per CTA, grid
// BH * p.num_pairs). tmQ8: e4m3 [B*Hq, N, d], 128-row boxes; tmK8/tmV8: e4m3
// [B*Hkv, N, d], 96-row boxes; 128B swizzle; tmO: bf16 output map as for the
// bf16 forward.
cudaError_t launch_mxfp8_quant(const MxParams& p, cudaStream_t stream);
cudaError_t launch_fwd_mxfp8(const CUtensorMap& tmQ8, const CUtensorMap& tmK8, const CUtensorMap& tmV8,
                             const CUtensorMap& tmO, const MxParams& p, int BH, bool causal, cudaStream_t stream);

struct DecParams {
  const uint16_t* q;  // bf16 [B*Hq, Nq, d]
  uint16_t* o;        // bf16 [B*Hq, Nq, d]
  float* lse;         // [B*Hq, Nq]
  float* o_part;      // workspace [ctas + B*Hkv, R, d] fp32, each normalised within its key range
  float* lse_part;    // workspace [ctas + B*Hkv, R], natural log (-inf: no visible key in the range)
  int* status;
  int Hq;
  int Hkv;
  int group;          // Hq / Hkv
  int Nq;
  int Nk;
  int R;              // group * Nq query rows per KV head
  int tiles;          // 64-key tiles per KV head: ceil(Nk / 64)
  int ctas;           // CTAs of the split pass (<= units)
  long long units;    // B * Hkv * tiles: the (KV head, key tile) work units
  int causal;
  float scale_log2;
};

// Decode-shaped forward. Split pass: CTA c takes the contiguous work units
// [c*units/ctas, (c+1)*units/ctas) in (KV head, key tile) order and writes one
// partial result per KV head it touches, to slot c + (b*Hkv + kv head). Then
// the log-sum-exp merge. tmK/tmV: bf16 [B*Hkv, Nk, d], 64 x 64 boxes, 128B
// swizzle.
cudaError_t launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecParams& p, int B, int d,
                          cudaStream_t stream);

// CTAs of the decode split pass that fit on the current device at once
// (0 if the device cannot be queried).
int decode_resident_ctas(int d);

}  // namespace fa
