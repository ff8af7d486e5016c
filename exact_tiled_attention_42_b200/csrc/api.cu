// The C ABI of include/fa.h: argument checks, TMA tensor maps, launches.
//
// Nothing here allocates device memory: every buffer, workspaces included,
// belongs to the caller. The only host-side state is the driver entry point
// for cuTensorMapEncodeTiled and the device address of the status word.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "kernels.h"

namespace {

__device__ int g_fa_status;  // first bounded-wait failure since it was last read

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Device address of g_fa_status on the current device (looked up once).
int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#ifdef FA_DEBUG_WITHHOLD
int g_debug_withhold = 0;  // debug build only: read by fa_fwd at each call
#endif

// Head dimensions: 64, 96 and 128 everywhere; 192 and 256 for the forward
// entry points (wide = true).
fa_status check_shape(int B, int Hq, int Hkv, int N, int d, float scale, bool wide = false) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 96 && d != 128 && !(wide && (d == 192 || d == 256))) return FA_ERR_UNSUPPORTED;
  // one 1-D grid of (batch x head) x (query or key tiles): must fit in 2^31 - 1
  const long long BH = static_cast<long long>(B) * Hq;
  const long long tiles = (N + 127) / 128;
  if (BH * tiles > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// 3-D map over a [rows_outer, N, d] bf16 tensor: box of 64 columns x box_rows rows.
bool make_map_bf16(CUtensorMap* m, const void* ptr, int d, int N, long long outer, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over a token-major packed [T, H, d] bf16 tensor: boxes of 64
// columns x 1 head x 128 tokens (the same 128-row x 128-byte shared-memory
// tile as make_map_bf16's).
bool make_map_bf16_packed(CUtensorMap* m, const void* ptr, int d, long long H, long long T, int box_rows = 128) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over the fp32 dQ accumulator [BH, N, d]: 16 x 32 boxes, 64B swizzle
// (the layout the backward's drain warps stage rows in).
bool make_map_f32_acc(CUtensorMap* m, const void* ptr, int d, int N, long long outer) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(N) * d * 4};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map over a packed fp32 dQ accumulator [T, Hq, d]: boxes of 16 columns
// x 1 head x 32 tokens, 64B swizzle (the drain's staging layout).
bool make_map_f32_acc_packed(CUtensorMap* m, const void* ptr, int d, long long H, long long T) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(H) * d * 4};
  cuuint32_t box[3] = {16, 1, 32};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
size_t up1024(size_t x) { return (x + 1023) & ~static_cast<size_t>(1023); }

// 3-D map over an e4m3 [outer, N, d] tensor: 128 x 128 boxes, 128B swizzle.
bool make_map_e4m3(CUtensorMap* m, const void* ptr, int d, int N, long long outer, int box_rows = 128) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N) * d};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Decode path: work units are (KV head, 64-key tile). Without a request the
// split pass runs as many CTAs as fit on the device at once, never more than
// the units or FA_DECODE_MAX_AUTO_CTAS (the bound the workspace is sized for).
constexpr long long FA_DECODE_MAX_AUTO_CTAS = 1024;

long long decode_units(int B, int Hkv, int Nk) { return static_cast<long long>(B) * Hkv * ((Nk + 63) / 64); }

// CTAs the workspace must cover (device independent)
long long decode_ctas_bound(long long units, int requested) {
  const long long want = requested > 0 ? requested : FA_DECODE_MAX_AUTO_CTAS;
  return want < units ? want : units;
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_BOUNDS: return "FA_ERR_BOUNDS";
  }
  return "FA_ERR_UNKNOWN";
}

#ifdef FA_DEBUG_WITHHOLD
// Debug build only (libfa_b200_debug.so, built with a 1 ms wait bound): while
// `on` is non-zero, fa_fwd's producer never issues its first V tile, so a
// bounded wait in every CTA runs out and reports FA_ERR_TIMEOUT. For the test
// of the abort path; the release library has no such switch.
void fa_debug_withhold_first_v(int on) { g_debug_withhold = on != 0; }
#endif

int fa_last_device_status(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(int)) != cudaSuccess) return -1;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  return v;
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int d, int causal, float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status st = check_shape(B, Hq, Hkv, N, d, scale, true);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  const bool wide = d > 128;  // 64-key tiles for K and V
  CUtensorMap tmQ, tmK, tmV, tmO;
  const long long BH = static_cast<long long>(B) * Hq, BHkv = static_cast<long long>(B) * Hkv;
  if (!make_map_bf16(&tmQ, q, d, N, BH, 128) || !make_map_bf16(&tmK, k, d, N, BHkv, wide ? 64 : 128) ||
      !make_map_bf16(&tmV, v, d, N, BHkv, wide ? 64 : 128) || !make_map_bf16(&tmO, o, d, N, BH, 128))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.lse = lse;
  p.status = status_ptr();
  p.cu_seqlens = nullptr;
  p.o = static_cast<uint16_t*>(o);
  p.total = 0;
  p.d = d;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.num_qtiles = (N + 127) / 128;
  p.num_pairs = (p.num_qtiles + 1) / 2;
  p.raster_heads = fa::raster_heads_for(BH, Hq / Hkv, 4ll * N * d);
  p.scale_log2 = scale * 1.4426950408889634f;
#ifdef FA_DEBUG_WITHHOLD
  p.debug_withhold = g_debug_withhold;
#endif
  if (!p.status) return FA_ERR_CUDA;
  cudaError_t e = wide ? fa::launch_fwd_wide(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), d, causal != 0, stream)
                       : fa::launch_fwd_bf16(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), d, causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal, float scale,
                        cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (total < 0 || max_seqlen < 0) return FA_ERR_INVALID_ARG;
  if (total == 0 || max_seqlen == 0) {  // every sequence is empty: nothing to compute
    fa_status st = check_shape(B, Hq, Hkv, 1, d, scale, true);
    return st;
  }
  fa_status st = check_shape(B, Hq, Hkv, max_seqlen, d, scale, true);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0)
    return FA_ERR_MISALIGNED;
  const bool wide = d > 128;
  CUtensorMap tmQ, tmK, tmV, tmO;
  if (!make_map_bf16_packed(&tmQ, q, d, Hq, total) || !make_map_bf16_packed(&tmK, k, d, Hkv, total, wide ? 64 : 128) ||
      !make_map_bf16_packed(&tmV, v, d, Hkv, total, wide ? 64 : 128) || !make_map_bf16_packed(&tmO, o, d, Hq, total))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.lse = lse;
  p.status = status_ptr();
  p.cu_seqlens = cu_seqlens;
  p.o = static_cast<uint16_t*>(o);
  p.total = total;
  p.d = d;
  p.N = max_seqlen;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.num_qtiles = (max_seqlen + 127) / 128;
  p.num_pairs = (p.num_qtiles + 1) / 2;
  p.raster_heads = fa::raster_heads_for(static_cast<long long>(B) * Hq, Hq / Hkv, 4ll * max_seqlen * d);
  p.scale_log2 = scale * 1.4426950408889634f;
#ifdef FA_DEBUG_WITHHOLD
  p.debug_withhold = 0;
#endif
  if (!p.status) return FA_ERR_CUDA;
  const long long BH = static_cast<long long>(B) * Hq;
  cudaError_t e = wide ? fa::launch_fwd_wide(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), d, causal != 0, stream)
                       : fa::launch_fwd_bf16(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), d, causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (check_shape(B, Hq, Hkv, N, d, 1.0f) != FA_OK) return 0;
  const size_t bh = static_cast<size_t>(B) * Hq;
  const size_t npad = static_cast<size_t>((N + 127) / 128) * 128;
  return 2 * up256(bh * npad * sizeof(float)) + up256(bh * N * d * sizeof(float));
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N,
                 int d, int causal, float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  fa_status st = check_shape(B, Hq, Hkv, N, d, scale);
  if (st != FA_OK) return st;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < fa_bwd_workspace_size(B, Hq, Hkv, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  const long long BH = static_cast<long long>(B) * Hq, BHkv = static_cast<long long>(B) * Hkv;
  const int T = (N + 127) / 128;

  const size_t vec_bytes = up256(static_cast<size_t>(BH) * T * 128 * sizeof(float));
  char* ws = static_cast<char*>(workspace);
  fa::BwdParams p;
  p.o = static_cast<const uint16_t*>(o);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.delta = reinterpret_cast<float*>(ws);
  p.neg_lse2 = reinterpret_cast<float*>(ws + vec_bytes);
  p.dq_accum = reinterpret_cast<float*>(ws + 2 * vec_bytes);
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.cu_seqlens = nullptr;
  p.total = 0;
  p.status = status_ptr();
  p.N = N;
  p.Npad = T * 128;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.num_tiles = T;
  p.d = d;
  p.d_pad = d == 64 ? 64 : 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (!p.status) return FA_ERR_CUDA;
  CUtensorMap tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmAcc;
  if (!make_map_bf16(&tmQ, q, d, N, BH, 128) || !make_map_bf16(&tmK, k, d, N, BHkv, 128) ||
      !make_map_bf16(&tmV, v, d, N, BHkv, 128) || !make_map_bf16(&tmdO, dout, d, N, BH, 128) ||
      !make_map_bf16(&tmdK, dk, d, N, BHkv, 128) || !make_map_bf16(&tmdV, dv, d, N, BHkv, 128) ||
      !make_map_f32_acc(&tmAcc, p.dq_accum, d, N, BH))
    return FA_ERR_CUDA;
  cudaError_t e = fa::launch_bwd_bf16(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmAcc, p, B, causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_varlen_workspace_size(int B, int Hq, int Hkv, int total, int max_seqlen, int d) {
  if (total < 0 || max_seqlen < 0 || check_shape(B, Hq, Hkv, max_seqlen > 0 ? max_seqlen : 1, d, 1.0f) != FA_OK)
    return 0;
  const size_t bh = static_cast<size_t>(B) * Hq;
  const size_t npad = static_cast<size_t>((max_seqlen + 127) / 128) * 128;
  const size_t ws = 2 * up256(bh * npad * sizeof(float)) + up256(static_cast<size_t>(total) * Hq * d * sizeof(float));
  return ws > 0 ? ws : 256;
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens, void* workspace,
                        size_t workspace_bytes, int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal,
                        float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !cu_seqlens) return FA_ERR_INVALID_ARG;
  if (total < 0 || max_seqlen < 0) return FA_ERR_INVALID_ARG;
  fa_status st = check_shape(B, Hq, Hkv, max_seqlen > 0 ? max_seqlen : 1, d, scale);
  if (st != FA_OK) return st;
  if (total == 0 || max_seqlen == 0) return FA_OK;  // every sequence is empty: nothing to compute
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < fa_bwd_varlen_workspace_size(B, Hq, Hkv, total, max_seqlen, d))
    return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  const long long BH = static_cast<long long>(B) * Hq;
  const int T = (max_seqlen + 127) / 128;
  const size_t vec_bytes = up256(static_cast<size_t>(BH) * T * 128 * sizeof(float));
  char* ws = static_cast<char*>(workspace);
  fa::BwdParams p;
  p.o = static_cast<const uint16_t*>(o);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.delta = reinterpret_cast<float*>(ws);
  p.neg_lse2 = reinterpret_cast<float*>(ws + vec_bytes);
  p.dq_accum = reinterpret_cast<float*>(ws + 2 * vec_bytes);
  p.dq = static_cast<uint16_t*>(dq);
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.cu_seqlens = cu_seqlens;
  p.total = total;
  p.status = status_ptr();
  p.N = max_seqlen;
  p.Npad = T * 128;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.num_tiles = T;
  p.d = d;
  p.d_pad = d == 64 ? 64 : 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (!p.status) return FA_ERR_CUDA;
  CUtensorMap tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmAcc;
  if (!make_map_bf16_packed(&tmQ, q, d, Hq, total) || !make_map_bf16_packed(&tmK, k, d, Hkv, total) ||
      !make_map_bf16_packed(&tmV, v, d, Hkv, total) || !make_map_bf16_packed(&tmdO, dout, d, Hq, total) ||
      !make_map_bf16_packed(&tmdK, dk, d, Hkv, total) || !make_map_bf16_packed(&tmdV, dv, d, Hkv, total) ||
      !make_map_f32_acc_packed(&tmAcc, p.dq_accum, d, Hq, total))
    return FA_ERR_CUDA;
  cudaError_t e = fa::launch_bwd_bf16(tmQ, tmK, tmV, tmdO, tmdK, tmdV, tmAcc, p, B, causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || num_ctas < 0 || (d != 64 && d != 128))
    return 0;
  const int R = (Hq / Hkv) * Nq;
  if (R > 16) return 0;
  const long long units = decode_units(B, Hkv, Nk);
  const size_t slots = static_cast<size_t>(decode_ctas_bound(units, num_ctas) + static_cast<long long>(B) * Hkv);
  const size_t rows = slots * R;
  return up256(rows * d * sizeof(float)) + up256(rows * sizeof(float));
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                        size_t workspace_bytes, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                        float scale, int num_ctas, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || Hq % Hkv != 0 || num_ctas < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal && Nk < Nq) return FA_ERR_INVALID_ARG;  // a query row would see no key
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * Nq > 16) return FA_ERR_UNSUPPORTED;  // query rows per KV head
  const long long BHkv = static_cast<long long>(B) * Hkv;
  const long long units = decode_units(B, Hkv, Nk);
  if (BHkv > 0x7fffffffLL || units > 0x7fffffffLL || static_cast<long long>(B) * Hq * Nq * 32 > 0x7fffffffLL)
    return FA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, lse};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
  const size_t need = fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_ctas);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  long long ctas = decode_ctas_bound(units, num_ctas);
  if (num_ctas == 0) {
    const int fit = fa::decode_resident_ctas(d);
    if (fit < 1) return FA_ERR_CUDA;
    if (fit < ctas) ctas = fit;
  }
  fa::DecParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.R = (Hq / Hkv) * Nq;
  // slots as sized by the workspace query; the kernels use the first ctas + B*Hkv
  const size_t slots = static_cast<size_t>(decode_ctas_bound(units, num_ctas) + BHkv);
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + up256(slots * p.R * d * sizeof(float)));
  p.status = status_ptr();
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.tiles = (Nk + 63) / 64;
  p.ctas = static_cast<int>(ctas);
  p.units = units;
  p.causal = causal != 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  if (!p.status) return FA_ERR_CUDA;
  CUtensorMap tmK, tmV;
  if (!make_map_bf16(&tmK, k, d, Nk, BHkv, 64) || !make_map_bf16(&tmV, v, d, Nk, BHkv, 64)) return FA_ERR_CUDA;
  cudaError_t e = fa::launch_decode(tmK, tmV, p, B, d, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_fp8_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (check_shape(B, Hq, Hkv, N, d, 1.0f) != FA_OK) return 0;
  const size_t nb = (N + 63) / 64;
  const size_t q = static_cast<size_t>(B) * Hq, kv = static_cast<size_t>(B) * Hkv;
  return up1024(q * N * d) + 2 * up1024(kv * N * d) + up1024(q * nb * 4) + 2 * up1024(kv * nb * 4);
}

}  // extern "C"

namespace {

// Validates the FP8 arguments shared by the three FP8 entry points and fills
// the parameter block (workspace layout: e4m3 Q, K, V codes, then the fp32
// block scales of Q, K, V, each region 1024-byte aligned).
fa_status fp8_setup(fa::Fp8Params* p, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
                    float scale, int use_rotation) {
  fa_status st = check_shape(B, Hq, Hkv, N, d, scale);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;  // the FP8 kernels are built for d = 128
  if (!workspace || workspace_bytes < fa_fp8_workspace_size(B, Hq, Hkv, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  const long long BH = static_cast<long long>(B) * Hq, BHkv = static_cast<long long>(B) * Hkv;
  const int nb = (N + 63) / 64;
  if (BH > 65535) return FA_ERR_UNSUPPORTED;  // pre-pass grid.y
  char* ws = static_cast<char*>(workspace);
  const size_t cq = up1024(static_cast<size_t>(BH) * N * d), ckv = up1024(static_cast<size_t>(BHkv) * N * d);
  const size_t sq = up1024(static_cast<size_t>(BH) * nb * 4), skv = up1024(static_cast<size_t>(BHkv) * nb * 4);
  p->src[0] = p->src[1] = p->src[2] = nullptr;
  p->codes[0] = reinterpret_cast<uint8_t*>(ws);
  p->codes[1] = reinterpret_cast<uint8_t*>(ws + cq);
  p->codes[2] = reinterpret_cast<uint8_t*>(ws + cq + ckv);
  p->scales[0] = reinterpret_cast<float*>(ws + cq + 2 * ckv);
  p->scales[1] = reinterpret_cast<float*>(ws + cq + 2 * ckv + sq);
  p->scales[2] = reinterpret_cast<float*>(ws + cq + 2 * ckv + sq + skv);
  p->heads[0] = static_cast<int>(BH);
  p->heads[1] = static_cast<int>(BHkv);
  p->heads[2] = static_cast<int>(BHkv);
  p->rotation_seed = 0;
  p->rotate = use_rotation != 0;
  p->lse = nullptr;
  p->N = N;
  p->nblk = nb;
  p->Hq = Hq;
  p->Hkv = Hkv;
  p->group = Hq / Hkv;
  p->num_qtiles = (N + 127) / 128;
  p->num_pairs = (p->num_qtiles + 1) / 2;
  p->raster_heads = fa::raster_heads_for(BH, Hq / Hkv, 2ll * N * d);  // e4m3 K and V
  p->score_log2 = scale * 1.4426950408889634f / (p->rotate ? static_cast<float>(d) : 1.0f);
  p->status = nullptr;  // set by the caller once every argument has been checked
  return FA_OK;
}

fa_status fp8_forward(const fa::Fp8Params& p, void* o, int B, int Hq, int Hkv, int N, int d, int causal,
                      cudaStream_t stream) {
  const long long BH = static_cast<long long>(B) * Hq, BHkv = static_cast<long long>(B) * Hkv;
  CUtensorMap tmQ, tmK, tmV, tmO;
  if (!make_map_e4m3(&tmQ, p.codes[0], d, N, BH) || !make_map_e4m3(&tmK, p.codes[1], d, N, BHkv) ||
      !make_map_e4m3(&tmV, p.codes[2], d, N, BHkv) || !make_map_bf16(&tmO, o, d, N, BH, 128))
    return FA_ERR_CUDA;
  cudaError_t e = fa::launch_fwd_fp8(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_fp8_quantize(const void* q, const void* k, const void* v, uint64_t rotation_seed, int use_rotation,
                          void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
                          cudaStream_t stream) {
  if (!q || !k || !v) return FA_ERR_INVALID_ARG;
  fa::Fp8Params p;
  fa_status st = fp8_setup(&p, workspace, workspace_bytes, B, Hq, Hkv, N, d, 1.0f, use_rotation);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return FA_ERR_MISALIGNED;
  p.src[0] = static_cast<const uint16_t*>(q);
  p.src[1] = static_cast<const uint16_t*>(k);
  p.src[2] = static_cast<const uint16_t*>(v);
  p.rotation_seed = rotation_seed;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  return fa::launch_fp8_quant(p, stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_fwd_fp8_quantized(const void* workspace, size_t workspace_bytes, void* o, float* lse, int use_rotation,
                               int B, int Hq, int Hkv, int N, int d, int causal, float scale, cudaStream_t stream) {
  if (!o || !lse) return FA_ERR_INVALID_ARG;
  fa::Fp8Params p;
  fa_status st = fp8_setup(&p, const_cast<void*>(workspace), workspace_bytes, B, Hq, Hkv, N, d, scale, use_rotation);
  if (st != FA_OK) return st;
  if (!aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  return fp8_forward(p, o, B, Hq, Hkv, N, d, causal, stream);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, uint64_t rotation_seed,
                     int use_rotation, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int N, int d,
                     int causal, float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa::Fp8Params p;
  fa_status st = fp8_setup(&p, workspace, workspace_bytes, B, Hq, Hkv, N, d, scale, use_rotation);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  p.src[0] = static_cast<const uint16_t*>(q);
  p.src[1] = static_cast<const uint16_t*>(k);
  p.src[2] = static_cast<const uint16_t*>(v);
  p.rotation_seed = rotation_seed;
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  if (fa::launch_fp8_quant(p, stream) != cudaSuccess) return FA_ERR_CUDA;
  return fp8_forward(p, o, B, Hq, Hkv, N, d, causal, stream);
}

}  // extern "C"

namespace {

// MXFP8 workspace: e4m3 codes of Q, K, V, then the exponent bytes of Q, K
// (4 per row) and V (vexp_stride per column: a 4-byte word per 96-key tile),
// each region 1024-byte aligned.
struct MxLayout {
  size_t cq, ckv, eq, ekv, ev;
  int num_ktiles, vexp_stride;
};
MxLayout mx_layout(int B, int Hq, int Hkv, int N, int d) {
  MxLayout L;
  L.num_ktiles = (N + 95) / 96;
  L.vexp_stride = 4 * L.num_ktiles;
  const size_t q = static_cast<size_t>(B) * Hq, kv = static_cast<size_t>(B) * Hkv;
  L.cq = up1024(q * N * d);
  L.ckv = up1024(kv * N * d);
  L.eq = up1024(q * N * 4);
  L.ekv = up1024(kv * N * 4);
  L.ev = up1024(kv * d * L.vexp_stride);
  return L;
}

}  // namespace

extern "C" {

size_t fa_mxfp8_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  if (check_shape(B, Hq, Hkv, N, d, 1.0f) != FA_OK || d != 128) return 0;
  const MxLayout L = mx_layout(B, Hq, Hkv, N, d);
  return L.cq + 2 * L.ckv + L.eq + L.ekv + L.ev;
}

fa_status fa_fwd_mxfp8(const void* q, const void* k, const void* v, void* o, float* lse, uint64_t rotation_seed,
                       int use_rotation, int scale_rule, void* workspace, size_t workspace_bytes, int B, int Hq,
                       int Hkv, int N, int d, int causal, float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status st = check_shape(B, Hq, Hkv, N, d, scale);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;  // built for d = 128
  if (scale_rule != 0 && scale_rule != 1) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < fa_mxfp8_workspace_size(B, Hq, Hkv, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  const long long BH = static_cast<long long>(B) * Hq, BHkv = static_cast<long long>(B) * Hkv;
  if (BH > 65535) return FA_ERR_UNSUPPORTED;  // pre-pass grid.y
  const MxLayout L = mx_layout(B, Hq, Hkv, N, d);
  char* ws = static_cast<char*>(workspace);
  fa::MxParams p;
  p.src[0] = static_cast<const uint16_t*>(q);
  p.src[1] = static_cast<const uint16_t*>(k);
  p.src[2] = static_cast<const uint16_t*>(v);
  p.codes[0] = reinterpret_cast<uint8_t*>(ws);
  p.codes[1] = reinterpret_cast<uint8_t*>(ws + L.cq);
  p.codes[2] = reinterpret_cast<uint8_t*>(ws + L.cq + L.ckv);
  p.exps[0] = reinterpret_cast<uint8_t*>(ws + L.cq + 2 * L.ckv);
  p.exps[1] = reinterpret_cast<uint8_t*>(ws + L.cq + 2 * L.ckv + L.eq);
  p.exps[2] = reinterpret_cast<uint8_t*>(ws + L.cq + 2 * L.ckv + L.eq + L.ekv);
  p.heads[0] = static_cast<int>(BH);
  p.heads[1] = static_cast<int>(BHkv);
  p.heads[2] = static_cast<int>(BHkv);
  p.rotation_seed = rotation_seed;
  p.rotate = use_rotation != 0;
  p.fit = scale_rule;
  p.lse = lse;
  p.status = status_ptr();
  p.N = N;
  p.num_ktiles = L.num_ktiles;
  p.vexp_stride = L.vexp_stride;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.group = Hq / Hkv;
  p.num_qtiles = (N + 127) / 128;
  p.num_pairs = (p.num_qtiles + 1) / 2;
  p.raster_heads = fa::raster_heads_for(BH, Hq / Hkv, 2ll * N * d);  // e4m3 K and V
  p.score_log2 = scale * 1.4426950408889634f / (p.rotate ? static_cast<float>(d) : 1.0f);
  if (!p.status) return FA_ERR_CUDA;
  CUtensorMap tmQ, tmK, tmV, tmO;
  if (!make_map_e4m3(&tmQ, p.codes[0], d, N, BH) || !make_map_e4m3(&tmK, p.codes[1], d, N, BHkv, 96) ||
      !make_map_e4m3(&tmV, p.codes[2], d, N, BHkv, 96) || !make_map_bf16(&tmO, o, d, N, BH, 128))
    return FA_ERR_CUDA;
  if (fa::launch_mxfp8_quant(p, stream) != cudaSuccess) return FA_ERR_CUDA;
  cudaError_t e = fa::launch_fwd_mxfp8(tmQ, tmK, tmV, tmO, p, static_cast<int>(BH), causal != 0, stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
