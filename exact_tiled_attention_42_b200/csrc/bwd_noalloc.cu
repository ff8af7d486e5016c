// fa_bwd_noalloc: the backward pass with its scratch memory built into the
// library, for callers that cannot allocate device memory themselves.
//
// fa_bwd needs a caller-provided workspace (D, -LSE log2 e and the fp32 dQ
// accumulator). Some callers have no way to provide one at the point of the
// call: plain C code with no device allocator of its own, or code that must
// not call cudaMalloc/cudaFree there because those calls synchronise the
// whole device (cudaFree always does) and would stall a stream-ordered
// pipeline. For them this entry point uses a fixed scratch array that lives
// in the library's device memory for as long as the library is loaded.
//
// The array is a file-scope __device__ symbol. In host code its name is only
// a host-side stand-in, never a device address, so its device address is
// looked up with cudaGetSymbolAddress once per device (with that device
// current), checked, cached, and passed on as the workspace of fa_bwd. That
// lookup happens on the first call on each device; make that first call
// before any stream capture. Nothing here allocates: no cudaMalloc, no
// cudaFree, no allocating library routine.
//
// Every call on a device shares the one array and leaves its contents
// behind. That is harmless here because the backward's preprocess rewrites
// every scratch value it later reads (D, -LSE log2 e, and zeros in the dQ
// accumulator) at the start of each call. Calls whose executions overlap on
// the GPU (different streams, or different host threads with no ordering
// between them) race on the array and give wrong results: serialise them.
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "fa.h"

namespace {

static __device__ __align__(256) unsigned char g_bwd_scratch[FA_BWD_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_bwd_scratch on the current device, or null on failure.
void* scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                    const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                                    int d, int causal, float scale, cudaStream_t stream) {
  // Argument errors first, in fa_bwd's order (null pointers, sizes, alignment),
  // so a call that is wrong in several ways reports the same error as fa_bwd;
  // only then the size limit of the built-in scratch.
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!ptr) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size(B, Hq, Hkv, N, d);
  if (need == 0) {
    // Invalid sizes: let fa_bwd's own checks report the precise error.
    return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, nullptr, 0, B, Hq, Hkv, N, d, causal, scale, stream);
  }
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
  if (need > FA_BWD_NOALLOC_MAX_BYTES) return FA_ERR_WORKSPACE;  // problem too large for the built-in scratch
  void* ws = scratch_ptr();
  if (!ws) return FA_ERR_CUDA;
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, ws, FA_BWD_NOALLOC_MAX_BYTES, B, Hq, Hkv, N, d, causal, scale,
                stream);
}
