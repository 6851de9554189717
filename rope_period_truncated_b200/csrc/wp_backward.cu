// WavePrune grouped-cutoff causal prefill: backward pass (dQ, dK, dV).
//
// What it computes: the gradients of sum(dO * O) through the forward
// definition (WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转周期",
// §2.1 Eq. (6), §2.3 Eq. (8)): with P_ij = exp(L_ij - LSE_i) from the
// forward's LSE and D_i = <dO_i, O_i>,
//   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (<dO_i, V_j> - D_i),
//   dQ_i[g] = scale * sum_j 1[i - j <= W_g] dS_ij K_j[g],
//   dK_j[g] = scale * sum_i 1[i - j <= W_g] dS_ij Q_i[g]   (16-dim group g).
// Three launches: delta_kernel below (D_i per row, fp32, into the caller's
// workspace), then the tensor-core dQ and dK/dV kernels of
// wp_backward_tc.cu. The logits are recomputed in both product kernels (7
// products per tile pair instead of 5) so that neither needs a cross-CTA
// reduction.
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_backward.h"
#include "wp_device.cuh"

namespace wp {

namespace {

constexpr int BWD_THREADS = 128;  // 4 warps

// ------------------------------------------------------------------ delta

template <int D>
__global__ void __launch_bounds__(BWD_THREADS) delta_kernel(const BackwardArgs a) {
  // one warp per (b, i, h) row, rows in [B, N, Hq] order
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (BWD_THREADS / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int64_t rows = static_cast<int64_t>(a.B) * a.N * a.Hq;
  if (row >= rows) return;
  const __nv_bfloat16 *o = a.o + row * D, *g = a.dout + row * D;
  float acc = 0.f;
  for (int e = lane; e < D; e += 32) acc = fmaf(__bfloat162float(o[e]), __bfloat162float(g[e]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const int64_t h = row % a.Hq, i = (row / a.Hq) % a.N, b = row / (static_cast<int64_t>(a.Hq) * a.N);
    a.delta[(b * a.Hq + h) * a.N + i] = acc;
  }
}

template <int D>
cudaError_t launch(const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(a.B) * a.N * a.Hq;
  delta_kernel<D><<<static_cast<unsigned>((rows + 3) / 4), BWD_THREADS, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_backward_dq_tc(D, a, maps, stream);
  if (e != cudaSuccess) return e;
  return launch_backward_dkdv_tc(D, a, maps, stream);
}

}  // namespace

cudaError_t launch_backward(int d_h, const BackwardArgs &a, const BackwardMaps &maps, cudaStream_t stream) {
  return d_h == 128 ? launch<128>(a, maps, stream) : launch<64>(a, maps, stream);
}

}  // namespace wp
