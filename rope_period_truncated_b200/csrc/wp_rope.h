// Internal launch interface of the RoPE kernel (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace wp {

struct RopeArgs {
  const __nv_bfloat16 *x;  // [tokens, H, D]
  __nv_bfloat16 *y;
  const int32_t *pos;      // [tokens] or null
  int64_t tokens;          // B * N
  int N, H;
  int64_t pos0;
  double freq[64];         // f_c, fp64, c < D/2
};

cudaError_t launch_rope(const RopeArgs &a, int d_h, int layout, cudaStream_t stream);

}  // namespace wp
