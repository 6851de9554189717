// WavePrune exact per-channel causal prefill (correctness path, CUDA cores).
//
// WavePrune reading notes "WavePrune：RoPE 通常只需一个旋转周期", §2.1 Eq. (6):
//   L_ij = scale * sum_c 1[i - j <= W_c] * (q_a k_a + q_b k_b),  j <= i,
// where (a, b) are the two dims of RoPE channel c; then the causal softmax
// and O = A V. A dropped channel adds 0, the pair stays in the softmax.
//
// One warp per query row: lanes take 32 keys at a time, each lane forms its
// key's logit channel by channel; the warp keeps an online softmax (row max
// and row sum by warp shuffles) and accumulates O with lanes over head dims.
// Not tuned for speed: the grouped tensor-core kernel is the fast path.
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_device.cuh"
#include "wp_prefill.h"

namespace wp {

namespace {

constexpr int ROWS_PER_CTA = 4;

template <int D>
__global__ void __launch_bounds__(ROWS_PER_CTA * 32) prefill_channel_kernel(const __grid_constant__ ChannelPrefillArgs a) {
  constexpr int C = D / 2;
  constexpr int PER_LANE = D / 32;
  __shared__ float q_s[ROWS_PER_CTA][D];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * ROWS_PER_CTA + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (a.Hq / a.Hkv);
  // Rows of this sequence: [b*N, b*N + N) of a uniform batch, or
  // [cu_seqlens[b], cu_seqlens[b+1]) of a packed one.
  int64_t N = a.N, row0 = static_cast<int64_t>(b) * a.N;
  if (a.cu_seqlens != nullptr) {
    row0 = a.cu_seqlens[b];
    const int64_t row1 = a.cu_seqlens[b + 1];
    if (row0 < 0 || row1 < row0 || row1 > a.T || row1 - row0 > a.N) {
      if (i == 0 && h == 0 && lane == 0) record_status(WP_ERR_ARG);
      return;
    }
    N = row1 - row0;
  }
  if (i >= N) return;
  const int32_t *cut = a.cut + (a.cut_rows == 1 ? 0 : h) * C;
  __nv_bfloat16 *orow = a.o + ((row0 + i) * a.Hq + h) * D;
  float *lse_at = a.lse == nullptr ? nullptr
                                   : a.lse + (a.cu_seqlens != nullptr ? static_cast<int64_t>(h) * a.T + row0 + i
                                                                      : (static_cast<int64_t>(b) * a.Hq + h) * a.N + i);
  if (*reinterpret_cast<volatile int *>(&g_status) != 0) {
    // A kernel of this library has given up since the status word was last
    // read: write NaN rows rather than leave stale outputs.
    for (int t = lane; t < D; t += 32) orow[t] = __ushort_as_bfloat16(0x7FC0);
    if (lane == 0 && lse_at != nullptr) *lse_at = __int_as_float(0x7FC00000);
    return;
  }
  const __nv_bfloat16 *qrow = a.q + ((row0 + i) * a.Hq + h) * D;
  for (int t = lane; t < D; t += 32) q_s[warp][t] = __bfloat162float(qrow[t]);
  __syncwarp();
  const int64_t kstride = static_cast<int64_t>(a.Hkv) * D;
  const __nv_bfloat16 *kbase = a.k + (row0 * a.Hkv + hk) * D;
  const __nv_bfloat16 *vbase = a.v + (row0 * a.Hkv + hk) * D;

  float m_run = -INFINITY, l_run = 0.f;
  float o[PER_LANE];
#pragma unroll
  for (int t = 0; t < PER_LANE; ++t) o[t] = 0.f;

  for (int64_t j0 = 0; j0 <= i; j0 += 32) {
    const int64_t j = j0 + lane;
    float s = -INFINITY;
    if (j <= i) {
      const __nv_bfloat16 *krow = kbase + j * kstride;
      const int64_t dist = i - j;
      float acc = 0.f;
      for (int c = 0; c < C; ++c) {
        if (dist > static_cast<int64_t>(cut[c])) continue;
        const int da = a.layout == WP_ROPE_INTERLEAVED ? 2 * c : c;
        const int db = a.layout == WP_ROPE_INTERLEAVED ? 2 * c + 1 : c + C;
        acc = fmaf(q_s[warp][da], __bfloat162float(krow[da]), acc);
        acc = fmaf(q_s[warp][db], __bfloat162float(krow[db]), acc);
      }
      s = acc * a.scale_log2;
    }
    float mx = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = exp2f(m_run - m_new);
    const float p = exp2f(s - m_new);
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l_run = l_run * alpha + ps;
    m_run = m_new;
#pragma unroll
    for (int t = 0; t < PER_LANE; ++t) o[t] *= alpha;
    const int nvalid = static_cast<int>(i - j0 + 1 < 32 ? i - j0 + 1 : 32);
    for (int kk = 0; kk < nvalid; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, p, kk);
      const __nv_bfloat16 *vrow = vbase + (j0 + kk) * kstride;
#pragma unroll
      for (int t = 0; t < PER_LANE; ++t) o[t] = fmaf(pk, __bfloat162float(vrow[lane + 32 * t]), o[t]);
    }
  }
  const float inv_l = 1.f / l_run;
#pragma unroll
  for (int t = 0; t < PER_LANE; ++t) orow[lane + 32 * t] = __float2bfloat16_rn(o[t] * inv_l);
  if (lane == 0 && lse_at != nullptr) *lse_at = (m_run + log2f(l_run)) * 0.69314718055994531f;
}

}  // namespace

cudaError_t launch_prefill_channel(int d_h, const ChannelPrefillArgs &a, cudaStream_t stream) {
  dim3 grid((a.N + ROWS_PER_CTA - 1) / ROWS_PER_CTA, a.Hq, a.B);
  if (d_h == 128)
    prefill_channel_kernel<128><<<grid, ROWS_PER_CTA * 32, 0, stream>>>(a);
  else
    prefill_channel_kernel<64><<<grid, ROWS_PER_CTA * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace wp
