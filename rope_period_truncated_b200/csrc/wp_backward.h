// Internal launch interface of the backward kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "wp_prefill.h"

namespace wp {

struct BackwardArgs {
  const __nv_bfloat16 *q, *k, *v, *o, *dout;  // q, o, dout [B, N, Hq, D]; k, v [B, N, Hkv, D]
  const float *lse;                           // [B, Hq, N], natural log (the forward's)
  float *delta;                               // [B, Hq, N]: rowsum(dout * o), written by the first kernel
  __nv_bfloat16 *dq, *dk, *dv;                // like q / k / v
  int B, N, Hq, Hkv;
  int cut_rows;                               // 1 or Hq
  float scale, scale_log2;
  int32_t cut[PREFILL_CUT_CAP];               // [cut_rows][D/16] group cutoffs
};

cudaError_t launch_backward(int d_h, const BackwardArgs &a, cudaStream_t stream);

}  // namespace wp
