// RoPE rotation of bf16 Q or K (memory-bound).
//
// kongchang.com page "WavePrune：RoPE只用一个旋转周期，长文本性能反而更好",
// RoPE paragraph: the pair of channel c at position m is multiplied by
// [[cos(m f_c), -sin(m f_c)], [sin(m f_c), cos(m f_c)]]; WavePrune reading
// notes "WavePrune：RoPE 通常只需一个旋转周期" §1.1: channel c of the token at
// position i rotates by i*f_c, f_c = theta^(-2c/d_h) times any frequency scale.
//
// One thread owns one token and 8 channels and walks all heads of that token,
// so each angle's sin/cos is formed once per token, not once per head. The
// angle p*f_c is formed and reduced modulo 2*pi in fp64 (p up to 2^31 and
// f_c near 1 would lose the phase in fp32), then sincosf on the reduced angle;
// the rotation is fp32 and the result rounds to bf16 (nearest even). Loads
// and stores are 16-byte vectors, coalesced along the head dim.
#include <cuda_bf16.h>
#include <cstdint>

#include "wp_rope.h"

namespace wp {

namespace {

constexpr int ROPE_THREADS = 256;

__device__ __forceinline__ void reduce_sincos(double ang, float *s, float *c) {
  constexpr double TWO_PI = 6.283185307179586476925286766559;
  constexpr double INV_TWO_PI = 0.15915494309189533576888376337251;
  const double k = rint(ang * INV_TWO_PI);
  const float r = static_cast<float>(fma(-k, TWO_PI, ang));
  sincosf(r, s, c);
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float2 v = __bfloat1622float2(h[t]);
    f[2 * t] = v.x;
    f[2 * t + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(f[2 * t], f[2 * t + 1]);
  return u;
}

// Interleaved: thread (token, chunk) owns dims [8*chunk, 8*chunk + 8), i.e.
// channels 4*chunk .. 4*chunk + 3 as adjacent (even, odd) pairs.
template <int D>
__global__ void __launch_bounds__(ROPE_THREADS) rope_interleaved_kernel(const RopeArgs a) {
  constexpr int CHUNKS = D / 8;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * ROPE_THREADS + threadIdx.x;
  const int64_t token = gid / CHUNKS;
  const int chunk = static_cast<int>(gid % CHUNKS);
  if (token >= a.tokens) return;
  const double p = a.pos ? static_cast<double>(a.pos[token]) : static_cast<double>(a.pos0 + token % a.N);
  float cs[4], sn[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) reduce_sincos(p * a.freq[4 * chunk + t], &sn[t], &cs[t]);
  const int64_t base = token * a.H * D + 8 * chunk;
  const uint4 *x = reinterpret_cast<const uint4 *>(a.x);
  uint4 *y = reinterpret_cast<uint4 *>(a.y);
#pragma unroll 4
  for (int hh = 0; hh < a.H; ++hh) {
    const int64_t off = (base + static_cast<int64_t>(hh) * D) / 8;
    float f[8], g[8];
    unpack8(x[off], f);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      g[2 * t] = f[2 * t] * cs[t] - f[2 * t + 1] * sn[t];
      g[2 * t + 1] = f[2 * t] * sn[t] + f[2 * t + 1] * cs[t];
    }
    y[off] = pack8(g);
  }
}

// Half-split: thread (token, chunk) owns channels [8*chunk, 8*chunk + 8),
// whose dims are [8*chunk, +8) and [C + 8*chunk, +8), C = D/2.
// PAIRED: write channel c's rotated pair to dims 2c, 2c+1 (the interleaved
// order) instead of back to c, c + D/2; then every 16-dim group holds 8 whole
// channels. Not in place (the writes land on other threads' inputs).
template <int D, bool PAIRED>
__global__ void __launch_bounds__(ROPE_THREADS) rope_half_split_kernel(const RopeArgs a) {
  constexpr int C = D / 2;
  constexpr int CHUNKS = C / 8;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * ROPE_THREADS + threadIdx.x;
  const int64_t token = gid / CHUNKS;
  const int chunk = static_cast<int>(gid % CHUNKS);
  if (token >= a.tokens) return;
  const double p = a.pos ? static_cast<double>(a.pos[token]) : static_cast<double>(a.pos0 + token % a.N);
  float cs[8], sn[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) reduce_sincos(p * a.freq[8 * chunk + t], &sn[t], &cs[t]);
  const int64_t base = token * a.H * D + 8 * chunk;
  const uint4 *x = reinterpret_cast<const uint4 *>(a.x);
  uint4 *y = reinterpret_cast<uint4 *>(a.y);
#pragma unroll 4
  for (int hh = 0; hh < a.H; ++hh) {
    const int64_t lo = (base + static_cast<int64_t>(hh) * D) / 8;
    const int64_t hi = lo + C / 8;
    float f[8], g[8], u[8], v[8];
    unpack8(x[lo], f);
    unpack8(x[hi], g);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      u[t] = f[t] * cs[t] - g[t] * sn[t];
      v[t] = f[t] * sn[t] + g[t] * cs[t];
    }
    if (PAIRED) {
      float w0[8], w1[8];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        w0[2 * t] = u[t];
        w0[2 * t + 1] = v[t];
        w1[2 * t] = u[t + 4];
        w1[2 * t + 1] = v[t + 4];
      }
      const int64_t out = (token * a.H * D + static_cast<int64_t>(hh) * D + 16 * chunk) / 8;
      y[out] = pack8(w0);
      y[out + 1] = pack8(w1);
    } else {
      y[lo] = pack8(u);
      y[hi] = pack8(v);
    }
  }
}

}  // namespace

cudaError_t launch_rope(const RopeArgs &a, int d_h, int layout, cudaStream_t stream) {
  const int chunks = layout == 0 ? d_h / 8 : d_h / 16;
  const int64_t threads = a.tokens * chunks;
  const int64_t blocks = (threads + ROPE_THREADS - 1) / ROPE_THREADS;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (layout == 0) {
    if (d_h == 128)
      rope_interleaved_kernel<128><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
    else
      rope_interleaved_kernel<64><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
  } else if (layout == 1) {
    if (d_h == 128)
      rope_half_split_kernel<128, false><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
    else
      rope_half_split_kernel<64, false><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
  } else {
    if (d_h == 128)
      rope_half_split_kernel<128, true><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
    else
      rope_half_split_kernel<64, true><<<static_cast<unsigned>(blocks), ROPE_THREADS, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace wp
