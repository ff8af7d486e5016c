// Launchers shared between the kernel translation units and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

struct FwdParams {
  float* lse;        // [B*Hq, N]
  int* status;       // device status word (bounded waits report here)
  int N;
  int Hq;
  int Hkv;
  int group;         // Hq / Hkv
  int num_qtiles;    // ceil(N / 128)
  int num_pairs;     // ceil(num_qtiles / 2): one CTA per pair of query tiles
  float scale_log2;  // scale * log2(e)
};

// tmQ/tmO: bf16 [B*Hq, N, d]; tmK/tmV: bf16 [B*Hkv, N, d]; all with
// 64-column x 128-row boxes and 128-byte swizzle.
cudaError_t launch_fwd_bf16(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const CUtensorMap& tmO, const FwdParams& p, int BH, int d, bool causal,
                            cudaStream_t stream);

}  // namespace fa
