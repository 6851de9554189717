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
  long long wait_limit;                       // bound of every mbarrier wait (tensor-core kernels)
  int32_t cut[PREFILL_CUT_CAP];               // [cut_rows][D/16] group cutoffs
};

// Tensor maps of the tensor-core backward kernels: 16-dim boxes with the
// 32-byte swizzle, 128 rows for the operands a CTA keeps (its own rows) and
// 64 rows for the streamed ones.
struct BackwardMaps {
  CUtensorMap q128, do128, k64, v64;  // dQ kernel
  CUtensorMap k128, v128, q64, do64;  // dK/dV kernel
};

cudaError_t launch_backward(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream);
cudaError_t launch_backward_dq_tc(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream);
cudaError_t launch_backward_dkdv_tc(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream);

}  // namespace wp
