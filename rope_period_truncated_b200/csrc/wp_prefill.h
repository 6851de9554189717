// Internal launch interface of the prefill kernels (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace wp {

struct PrefillArgs {
  __nv_bfloat16 *o;  // [B, N, Hq, D]
  float *lse;        // [B, Hq, N] or null
  int B, N, Hq, Hkv;
  int32_t cut[8];    // group cutoffs, D/16 entries
  float scale_log2;  // softmax scale * log2(e)
  long long wait_limit;
};

struct ChannelPrefillArgs {
  const __nv_bfloat16 *q, *k, *v;  // [B, N, H, D]
  __nv_bfloat16 *o;
  float *lse;
  int B, N, Hq, Hkv, layout;
  int32_t cut[64];  // channel cutoffs, D/2 entries
  float scale_log2;
};

cudaError_t launch_prefill_grouped(int d_h, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                   const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_channel(int d_h, const ChannelPrefillArgs &a, cudaStream_t stream);

}  // namespace wp
